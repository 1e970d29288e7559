"""GPU decode step vs the CPU oracle, through the C ABI, teacher-forced on seeded inputs."""
import os

import numpy as np
import pytest

import fixtures as fx
from tests.gpu_harness import assert_parity, run_teacher_forced

pytestmark = pytest.mark.gpu


def test_tiny_all_steps():
    res = run_teacher_forced(fx.CONFIGS["tiny"])
    assert_parity(res)


@pytest.mark.parametrize("kw,gains", [
    ({"qk_norm": True, "tied_embeddings": True, "rope_theta": 5e5}, "random"),
    ({"ctx": 0, "steps": 3}, "ones"),                      # empty cache: position 0
    ({"ctx": 255, "steps": 3}, "random"),                  # new token crosses a chunk boundary
    ({"n_q_heads": 8, "n_kv_heads": 1}, "ones"),           # 8 query heads per KV head
    ({"n_q_heads": 2, "n_kv_heads": 2}, "ones"),           # MHA
    ({"ffn_dim": 5920, "steps": 3}, "random"),             # > 32 neurons per SM: gate and up as two stage groups
])
def test_tiny_variants(kw, gains):
    res = run_teacher_forced(fx.CONFIGS["tiny"].replace(**kw), steps=kw.get("steps", 4), gains=gains)
    assert_parity(res)


def test_tiny_head_dim_128_small_units(monkeypatch):
    monkeypatch.setenv("MK_ATTN_UNIT", "40")             # 40-position units: rows cut into many pieces
    cfg = fx.CONFIGS["tiny"].replace(n_q_heads=4, n_kv_heads=2, head_dim=128, ctx=200, steps=3)
    assert_parity(run_teacher_forced(cfg, gains="random"))


def test_tiny_last_cache_slot():
    cfg = fx.CONFIGS["tiny"].replace(ctx=141, steps=3)   # writes slots 141..143 of 144
    assert_parity(run_teacher_forced(cfg))


def test_dense_0_6b_all_steps():
    """The 0.6B shape (qk-norm, tied embeddings) end to end over all 64 of its decode steps."""
    assert_parity(run_teacher_forced(fx.CONFIGS["dense-0.6b"]))


# ---- paged KV cache through the oracle ---------------------------------------------------------

@pytest.mark.parametrize("kw,gains", [
    ({"n_q_heads": 4, "n_kv_heads": 2, "head_dim": 128, "ctx": 200, "steps": 4}, "random"),           # batch 1
    ({"n_q_heads": 8, "n_kv_heads": 2, "head_dim": 128, "batch": 3, "ffn_dim": 704, "ctx": 0, "ctx_lo": 5,
      "ctx_hi": 260, "steps": 3}, "random"),                                                          # tensor cores
    ({"n_q_heads": 4, "n_kv_heads": 2, "head_dim": 128, "batch": 2, "ffn_dim": 0, "n_experts": 8, "top_k": 2,
      "expert_ffn_dim": 128, "ctx": 0, "ctx_lo": 100, "ctx_hi": 300, "steps": 3}, "random"),          # MoE
])
def test_paged_cache_against_the_oracle(kw, gains):
    """Every sequence's cache in a shuffled page pool (spare pages NaN): the oracle keeps its own
    contiguous cache, the GPU reads and appends through the block table."""
    cfg = fx.CONFIGS["tiny"].replace(**kw)
    res = run_teacher_forced(cfg, gains=gains, paged=True)
    assert_parity(res)


# ---- batch > 1 (tensor-core projections) -------------------------------------------------------

# the batched GEMV reads K in blocks of 64 columns: tiny's ffn width 688 becomes 704
@pytest.mark.parametrize("kw,gains", [
    ({"batch": 4, "ctx": 0, "ctx_lo": 3, "ctx_hi": 60, "steps": 3}, "random"),
    ({"batch": 8, "ctx": 0, "steps": 2}, "ones"),                                    # empty caches
    ({"batch": 2, "n_q_heads": 8, "n_kv_heads": 1, "qk_norm": True, "tied_embeddings": True}, "random"),
    ({"batch": 3, "ctx": 0, "ctx_lo": 250, "ctx_hi": 260, "steps": 3}, "ones"),    # chunk boundary, ragged
])
def test_tiny_batched(kw, gains):
    cfg = fx.CONFIGS["tiny"].replace(ffn_dim=704, **kw)
    assert_parity(run_teacher_forced(cfg, steps=kw.get("steps", 3), gains=gains))


def test_batched_small_units(monkeypatch):
    # tensor-core attention with 24-position units: every stage box carries
    # positions past the piece (masked keys, zeroed values) and rows span many slots
    monkeypatch.setenv("MK_ATTN_UNIT", "24")
    cfg = fx.CONFIGS["tiny"].replace(ffn_dim=704, batch=5, ctx=0, ctx_lo=1, ctx_hi=140, steps=3)
    assert_parity(run_teacher_forced(cfg, gains="random"))


def test_batched_multi_chunk():
    # MHA, head_dim 128; the down projection (K = 4608) streams 5 column chunks,
    # the last one half empty (its TMA boxes read zeros past K); hidden = 640
    # leaves 24 of each chunk's 64 k-steps idle
    cfg = fx.ModelConfig("mid-b8", n_layers=3, hidden=640, n_q_heads=5, n_kv_heads=5, head_dim=128, ffn_dim=4608,
                         vocab=2000, batch=8, ctx_lo=10, ctx_hi=300, steps=3)
    assert_parity(run_teacher_forced(cfg, gains="random"))


# ---- mixture of experts (tensor-core kernel at any batch size) -------------------------------------

@pytest.mark.parametrize("kw,gains", [
    ({"n_experts": 8, "top_k": 2, "expert_ffn_dim": 128, "batch": 4, "ctx": 0, "ctx_lo": 3, "ctx_hi": 120}, "random"),
    ({"n_experts": 16, "top_k": 4, "expert_ffn_dim": 64, "batch": 1}, "ones"),                      # MoE at batch 1
    ({"n_experts": 32, "top_k": 8, "expert_ffn_dim": 64, "batch": 8, "ctx": 0, "ctx_lo": 0, "ctx_hi": 60}, "random"),
    ({"n_experts": 256, "top_k": 8, "expert_ffn_dim": 1088, "batch": 3, "n_layers": 1}, "random"),   # ragged Ie chunk
])
def test_tiny_moe(kw, gains):
    cfg = fx.CONFIGS["tiny"].replace(ffn_dim=0, **kw)
    res = run_teacher_forced(cfg, steps=3, gains=gains)
    assert_parity(res)
    assert len(res["sel_own"]) == 3 * cfg.n_layers * cfg.batch
