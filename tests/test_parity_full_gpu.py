"""Parity at the full 8B, 13B batch-8 and MoE shapes, over every decode step of each workload.

The GPU runs all of the workload's teacher-forced steps (8B: 128, 13B batch 8:
64, MoE: 32) in the configuration bench.py times.  Then the oracle checks:

* every step: the LM head and top-1 pick, recomputed from the GPU's own final
  residual of that step (logits max-abs; exact arg-max on the batch-1 kernel,
  the tie reading of tests/gpu_harness.py on the tensor-core kernel);
* the first, middle and last step: sampled layers recomputed one by one from
  the GPU's own input to the layer (its dumped residual) and the GPU's own
  cache at that step (the generator's prefill plus the rows the GPU appended
  at earlier steps): hidden states after attention and after the MLP, the
  appended K/V rows, and for MoE the routing checks (i)-(iii).  A sequence
  whose MoE pick set differs from the oracle's (allowed only at a near-tie of
  the router logits) ran other experts: its MLP output is left out of that
  layer's hidden-state comparison.

Each check is independent of the others, so error cannot hide in a growing
residual.  Tolerances as in tests/gpu_harness.py.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import fixtures as fx
import oracle as ora
from fixtures.device import device_caches, device_model
from tests.gpu_harness import (MIN_TOP1, TOL_HIDDEN, TOL_KV, TOL_LOGITS_ABS, bits, log_result, tensor_core_kernel,
                               top1_agree, top1_exact)
from tests.helpers import bf16_f64, expert_loader, host_model, rel_l2

pytestmark = pytest.mark.gpu


def run_all_steps(cfg, layers):
    """GPU over all cfg.steps steps; host copies of what the oracle checks."""
    import auto_regressive_decode_b200.mk as mk
    S0 = fx.context_lengths(cfg)
    toks = fx.tokens(cfg)
    w = device_model(cfg)
    kc, vc = device_caches(cfg, S0)
    dec = mk.Decoder(cfg, w, kc, vc)
    B, L, T = cfg.batch, cfg.n_layers, cfg.steps
    sampled = sorted({0, T // 2, T - 1})
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    out = {"S0": S0, "toks": toks, "final": [], "logits": [], "snap": {}, "sampled": sampled}
    for t in range(T):
        S = torch.from_numpy((S0 + t).astype(np.int32)).cuda()
        dec.step(torch.from_numpy(toks[t].copy()).cuda(), S, S, logits)
        assert dec.status() == mk.MK_OK, t
        hid = dec.hidden_states()
        out["final"].append(hid[2 * L].cpu().numpy().astype(np.float64))
        out["logits"].append(logits.cpu().numpy().astype(np.float64))
        if t in sampled:
            out["snap"][t] = {"hid": hid.cpu().numpy().astype(np.float64),
                              "routing": dec.routing() if cfg.n_experts else None}
    # the rows the GPU appended, per sampled layer: [B][nkv][T][hd] (bf16 bits)
    out["k_rows"] = {l: np.stack([bits(kc[l, b, :, S0[b]:S0[b] + T].contiguous()) for b in range(B)])
                     for l in layers}
    out["v_rows"] = {l: np.stack([bits(vc[l, b, :, S0[b]:S0[b] + T].contiguous()) for b in range(B)])
                     for l in layers}
    dec.close()
    del w, kc, vc
    torch.cuda.empty_cache()
    return out


def check_layers(cfg, run, model, layers):
    """Sampled layers at the first, middle and last step, from the GPU's own inputs and cache."""
    S0, B = run["S0"], cfg.batch
    for t in run["sampled"]:
        hid = run["snap"][t]["hid"]
        S = (S0 + t).astype(np.int32)
        for l in layers:
            okc = fx.kv_prefill(cfg, l, 0, S0)
            ovc = fx.kv_prefill(cfg, l, 1, S0)
            for b in range(B):   # the rows the GPU appended before step t
                okc[b, :, S0[b]:S0[b] + t] = run["k_rows"][l][b][:, :t]
                ovc[b, :, S0[b]:S0[b] + t] = run["v_rows"][l][b][:, :t]
            o = model.layer_forward(l, hid[2 * l].copy(), okc, ovc, S, S)
            if cfg.n_experts:
                model.clear_expert_cache()
            assert rel_l2(hid[2 * l + 1], o["h_attn"]) <= TOL_HIDDEN, (t, l)
            # MLP output: the sequences whose experts are the oracle's (a sequence
            # whose pick set differs, at a near-tie only (check_moe_layer), ran other
            # experts and has no comparable output)
            rows = check_moe_layer(cfg, run["snap"][t]["routing"], o, l, t) if cfg.n_experts else list(range(B))
            assert rel_l2(hid[2 * l + 2][rows], o["h_mlp"][rows]) <= TOL_HIDDEN, (t, l, rows)
            for b in range(B):
                gk = bf16_f64(run["k_rows"][l][b][:, t])
                gv = bf16_f64(run["v_rows"][l][b][:, t])
                assert rel_l2(gk, bf16_f64(okc[b, :, S[b]])) <= TOL_KV, (t, l, b)
                assert rel_l2(gv, bf16_f64(ovc[b, :, S[b]])) <= TOL_KV, (t, l, b)


def check_moe_layer(cfg, routing, o, l, t):
    """(ii) router logits; (iii) end-to-end pick sets differ only at near-ties.  Returns the
    sequences whose pick set is the oracle's."""
    r, sel, sw, n = routing
    assert rel_l2(r[l].astype(np.float64), o["router_logits"]) <= TOL_HIDDEN, (t, l)
    same = []
    for b in range(cfg.batch):
        if set(sel[l, b].tolist()) != set(o["sel"][b].tolist()):
            srt = np.sort(o["router_logits"][b])[::-1]
            err = float(np.max(np.abs(r[l, b] - o["router_logits"][b])))
            assert srt[cfg.top_k - 1] - srt[cfg.top_k] < 2 * err, (t, l, b)
        else:
            same.append(b)
    assert same, (t, l)
    return same


def check_routing_every_layer(cfg, run):
    """(i) at the sampled steps, on every layer: the picks are the oracle's top-k of the GPU's router logits."""
    for t in run["sampled"]:
        r, sel, sw, n = run["snap"][t]["routing"]
        for l in range(cfg.n_layers):
            assert int(n[l]) == len(np.unique(sel[l])), (t, l)
            for b in range(cfg.batch):
                own, own_w = ora.topk(r[l, b].astype(np.float64), cfg.top_k)
                assert np.array_equal(sel[l, b], own), (t, l, b)
                assert float(np.max(np.abs(sw[l, b] - own_w))) <= 1e-5, (t, l, b)


def check_logits_every_step(cfg, run, model):
    """LM head of every step from the GPU's final residual (oracle calls in threads: the C call drops the GIL)."""
    T, B = cfg.steps, cfg.batch
    jobs = [(t, b) for t in range(T) for b in range(B)]
    with ThreadPoolExecutor(max_workers=16) as ex:
        refs = list(ex.map(lambda tb: model.lm_head(run["final"][tb[0]][tb[1]]), jobs))
    ref = np.stack(refs).reshape(T, B, cfg.vocab)
    gpu = np.stack(run["logits"])[:, :B]
    assert float(np.max(np.abs(gpu - ref))) <= TOL_LOGITS_ABS
    exact = [e for t in range(T) for e in top1_exact(gpu[t], ref[t])]
    tie = [e for t in range(T) for e in top1_agree(gpu[t], ref[t])]
    pick = np.argmax(gpu, axis=2)
    got = np.take_along_axis(ref, pick[..., None], axis=2)[..., 0]
    gaps = (ref.max(axis=2) - got)[pick != np.argmax(ref, axis=2)]
    log_result({"config": cfg.name, "kernel": "tensor-core" if tensor_core_kernel(cfg) else "cuda-core",
                "paged": False, "top1_exact": exact, "top1": tie, "top1_gaps": [float(g) for g in gaps],
                "hidden": [0.0], "logits_abs": [float(np.max(np.abs(gpu - ref)))], "kv": [0.0], "router": []})
    if tensor_core_kernel(cfg):
        assert np.mean(tie) >= MIN_TOP1, (np.mean(tie), np.mean(exact))
    else:
        assert np.mean(exact) >= MIN_TOP1, (np.mean(exact), gaps)


def test_dense_8b_all_steps():
    """8B shape, batch 1, context 4096, 128 steps (the batch-1 CUDA-core kernel)."""
    cfg = fx.CONFIGS["dense-8b"]
    layers = (0, 13, 31)
    run = run_all_steps(cfg, layers)
    g, ls = host_model(cfg, layers=layers)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls)
    for t in run["sampled"]:   # the embedding row enters bit-exact
        assert np.array_equal(run["snap"][t]["hid"][0, 0], bf16_f64(g["embed"][run["toks"][t][0]]))
    check_layers(cfg, run, model, layers)
    check_logits_every_step(cfg, run, model)


def test_dense_13b_batch8_ragged_all_steps():
    """13B shape, batch 8 with ragged contexts in [256, 4096], 64 steps: tensor-core projections."""
    cfg = fx.CONFIGS["dense-13b-b8"]
    layers = (0, 39)
    run = run_all_steps(cfg, layers)
    g, ls = host_model(cfg, layers=layers)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls)
    check_layers(cfg, run, model, layers)
    check_logits_every_step(cfg, run, model)


def test_moe_128x8_all_steps():
    """MoE shape: 48 layers, 128 experts, top-8, batch 4, contexts in [512, 2048], 32 steps."""
    cfg = fx.CONFIGS["moe-128x8"]
    layers = (0, 23, 47)
    run = run_all_steps(cfg, layers)
    check_routing_every_layer(cfg, run)
    g, ls = host_model(cfg, layers=layers)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls, expert_loader(cfg))
    check_layers(cfg, run, model, layers)
    check_logits_every_step(cfg, run, model)
