"""bench.py's algorithmic bytes (the roofline numerator) against the model's own tensor list.

The bytes a step must move are every bf16 weight it reads once (all layer tensors, the LM head, the
batch's embedding rows; MoE: the router and only the distinct picked experts) plus the KV positions
it reads and the row it appends.  Here they are summed tensor by tensor from the seeded generator's
recipe (fixtures), independently of bench.py's closed form.
"""
import numpy as np
import pytest

import bench
import fixtures as fx


def _numel(spec):
    return int(np.prod(spec.shape))


@pytest.mark.parametrize("name", ["tiny", "dense-0.6b", "dense-8b", "dense-13b-b8", "moe-128x8"])
def test_weight_bytes_match_the_tensor_list(name):
    cfg = fx.CONFIGS[name]
    total = 0
    for l in range(cfg.n_layers):
        total += sum(_numel(s) for s in fx.layer_specs(cfg, l).values())
    g = fx.global_specs(cfg)
    total += _numel(g["final_norm"])
    total += cfg.batch * cfg.hidden                       # the batch's embedding rows
    if cfg.tied_embeddings:
        total += _numel(g["embed"])                       # the LM head is the embedding matrix
    else:
        total += _numel(g["lm_head"])
    assert bench.weight_bytes_read(cfg) == 2 * total


def test_kv_bytes_closed_form():
    cfg = fx.CONFIGS["dense-8b"]
    # K and V, 32 layers x 8 heads x 128 dims x 2 bytes, 4096 cached positions read + 1 appended
    assert bench.kv_bytes(cfg, [4096]) == 2 * 32 * 8 * 128 * 2 * 4097
    cfg = fx.CONFIGS["dense-13b-b8"]
    lens = [10, 0, 4095]
    assert bench.kv_bytes(cfg, lens) == 2 * 40 * 40 * 128 * 2 * (11 + 1 + 4096)


def test_expert_bytes_count_distinct_experts_once():
    cfg = fx.CONFIGS["moe-128x8"]
    one = sum(_numel(s) for s in fx.expert_specs(cfg, 0, 0).values()) * 2
    assert bench.expert_bytes_read(cfg, [29.0]) == pytest.approx(29 * one)
    assert bench.expert_bytes_read(cfg, [28, 30]) == pytest.approx(29 * one)   # mean over the steps


def test_8b_step_bytes():
    # the headline workload at 4096 cached positions: weights 15.0099 GB + KV 0.5370 GB = 15.5469 GB
    # (bench.py averages the KV part over its timed steps, whose lengths grow from 4096)
    cfg = fx.CONFIGS["dense-8b"]
    b = bench.weight_bytes_read(cfg) + bench.kv_bytes(cfg, fx.context_lengths(cfg))
    assert b == 15_009_857_536 + 537_001_984


def test_traffic_is_reported_only_for_the_captured_kernel_source(tmp_path, monkeypatch):
    """`roofline.traffic` comes from profiles/traffic.json only while that capture's kernel source hash is
    the current one; every committed entry is a whole-workload figure scaled from its small case."""
    import json
    d = json.load(open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for name, e in d.items():
        assert name in fx.CONFIGS
        ratio = e["traffic_over_algorithmic"]
        assert 1.0 <= ratio < 1.05, name                          # no re-reads beyond whole attention stages
        assert abs(e["dram_bytes_per_launch"] - ratio * e["algorithmic_full"]) <= 1e-5 * e["algorithmic_full"]  # ratio kept to 5 digits
        assert e["algorithmic_small"] < e["algorithmic_full"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "not-the-captured-source")
    assert bench.ncu_traffic("dense-8b") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: d["dense-8b"]["kernel_source"])
    assert bench.ncu_traffic("dense-8b") == d["dense-8b"]["dram_bytes_per_launch"]
