"""Parity at the full 8B, 13B batch-8 and MoE shapes, in the configurations bench.py times.

The whole step runs on the GPU; the oracle then recomputes sampled layers one by
one from the GPU's own input to each layer (its dumped residual), and the LM
head from the GPU's final residual, so each check is independent of the
others.  Tolerances as in tests/gpu_harness.py.
"""
import numpy as np
import pytest
import torch

import fixtures as fx
import oracle as ora
from fixtures.device import device_caches, device_model
from tests.gpu_harness import TOL_HIDDEN, TOL_KV, TOL_LOGITS_ABS, bits, top1_agree
from tests.helpers import bf16_f64, expert_loader, host_model, rel_l2

pytestmark = pytest.mark.gpu

SAMPLED_LAYERS = (0, 13, 31)


def test_dense_8b_sampled_layers_and_logits():
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["dense-8b"]
    S0 = fx.context_lengths(cfg)
    tok = fx.tokens(cfg)[0]
    w = device_model(cfg)
    kc, vc = device_caches(cfg, S0)
    dec = mk.Decoder(cfg, w, kc, vc)
    logits = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    d_tok = torch.from_numpy(tok.copy()).cuda()
    d_len = torch.from_numpy(S0.copy()).cuda()
    dec.step(d_tok, d_len, d_len, logits)
    assert dec.status() == mk.MK_OK
    hid = dec.hidden_states().cpu().numpy().astype(np.float64)
    lg = logits.cpu().numpy().astype(np.float64)[0]
    S = int(S0[0])
    k_new = {l: bf16_f64(bits(kc[l, 0, :, S].contiguous())) for l in SAMPLED_LAYERS}
    v_new = {l: bf16_f64(bits(vc[l, 0, :, S].contiguous())) for l in SAMPLED_LAYERS}
    dec.close()
    del w, kc, vc
    torch.cuda.empty_cache()

    g, ls = host_model(cfg, layers=SAMPLED_LAYERS)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls)
    assert np.array_equal(hid[0, 0], bf16_f64(g["embed"][tok[0]]))
    for l in SAMPLED_LAYERS:
        okc = fx.kv_prefill(cfg, l, 0, S0)
        ovc = fx.kv_prefill(cfg, l, 1, S0)
        out = model.layer_forward(l, hid[2 * l].copy(), okc, ovc, S0, S0)
        assert rel_l2(hid[2 * l + 1], out["h_attn"]) <= TOL_HIDDEN, l
        assert rel_l2(hid[2 * l + 2], out["h_mlp"]) <= TOL_HIDDEN, l
        assert rel_l2(k_new[l], bf16_f64(okc[0, :, S])) <= TOL_KV, l
        assert rel_l2(v_new[l], bf16_f64(ovc[0, :, S])) <= TOL_KV, l
    ref = model.lm_head(hid[2 * cfg.n_layers, 0])
    assert float(np.max(np.abs(lg - ref))) <= TOL_LOGITS_ABS
    assert all(top1_agree(lg[None], ref[None]))


def test_dense_13b_batch8_ragged_sampled_layers_and_logits():
    """13B shape, batch 8 with ragged contexts in [256, 4096]: tensor-core projections."""
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["dense-13b-b8"]
    S0 = fx.context_lengths(cfg)
    tok = fx.tokens(cfg)[0]
    w = device_model(cfg)
    kc, vc = device_caches(cfg, S0)
    dec = mk.Decoder(cfg, w, kc, vc)
    logits = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    d_tok = torch.from_numpy(tok.copy()).cuda()
    d_len = torch.from_numpy(S0.copy()).cuda()
    dec.step(d_tok, d_len, d_len, logits)
    assert dec.status() == mk.MK_OK
    hid = dec.hidden_states().cpu().numpy().astype(np.float64)
    lg = logits.cpu().numpy().astype(np.float64)
    layers = (0, 39)
    new_rows = {}
    for l in layers:
        for b in range(cfg.batch):
            S = int(S0[b])
            new_rows[(l, b)] = (bf16_f64(bits(kc[l, b, :, S].contiguous())), bf16_f64(bits(vc[l, b, :, S].contiguous())))
    dec.close()
    del w, kc, vc
    torch.cuda.empty_cache()

    g, ls = host_model(cfg, layers=layers)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls)
    for l in layers:
        okc = fx.kv_prefill(cfg, l, 0, S0)
        ovc = fx.kv_prefill(cfg, l, 1, S0)
        out = model.layer_forward(l, hid[2 * l].copy(), okc, ovc, S0, S0)
        assert rel_l2(hid[2 * l + 1], out["h_attn"]) <= TOL_HIDDEN, l
        assert rel_l2(hid[2 * l + 2], out["h_mlp"]) <= TOL_HIDDEN, l
        for b in range(cfg.batch):
            S = int(S0[b])
            assert rel_l2(new_rows[(l, b)][0], bf16_f64(okc[b, :, S])) <= TOL_KV
            assert rel_l2(new_rows[(l, b)][1], bf16_f64(ovc[b, :, S])) <= TOL_KV
    refs = np.stack([model.lm_head(hid[2 * cfg.n_layers, b]) for b in range(cfg.batch)])
    assert float(np.max(np.abs(lg[:cfg.batch] - refs))) <= TOL_LOGITS_ABS
    assert all(top1_agree(lg[:cfg.batch], refs))


def test_moe_128x8_sampled_layers_routing_and_logits():
    """MoE shape: 48 layers, 128 experts, top-8, batch 4, contexts in [512, 2048]."""
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["moe-128x8"]
    S0 = fx.context_lengths(cfg)
    tok = fx.tokens(cfg)[0]
    w = device_model(cfg)
    kc, vc = device_caches(cfg, S0)
    dec = mk.Decoder(cfg, w, kc, vc)
    logits = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    d_tok = torch.from_numpy(tok.copy()).cuda()
    d_len = torch.from_numpy(S0.copy()).cuda()
    dec.step(d_tok, d_len, d_len, logits)
    assert dec.status() == mk.MK_OK
    hid = dec.hidden_states().cpu().numpy().astype(np.float64)
    r, sel, sw, n = dec.routing()
    lg = logits.cpu().numpy().astype(np.float64)
    layers = (0, 23, 47)
    dec.close()
    del w, kc, vc
    torch.cuda.empty_cache()

    # (i) on every layer: the picks are the oracle's top-k of the GPU's own router logits
    for l in range(cfg.n_layers):
        assert int(n[l]) == len(np.unique(sel[l]))
        for b in range(cfg.batch):
            own, own_w = ora.topk(r[l, b].astype(np.float64), cfg.top_k)
            assert np.array_equal(sel[l, b], own), (l, b)
            assert float(np.max(np.abs(sw[l, b] - own_w))) <= 1e-5
    g, ls = host_model(cfg, layers=layers)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls, expert_loader(cfg))
    for l in layers:
        okc = fx.kv_prefill(cfg, l, 0, S0)
        ovc = fx.kv_prefill(cfg, l, 1, S0)
        out = model.layer_forward(l, hid[2 * l].copy(), okc, ovc, S0, S0)
        model.clear_expert_cache()
        assert rel_l2(hid[2 * l + 1], out["h_attn"]) <= TOL_HIDDEN, l
        assert rel_l2(hid[2 * l + 2], out["h_mlp"]) <= TOL_HIDDEN, l
        # (ii) router logits; (iii) end-to-end pick sets differ only at near-ties
        assert rel_l2(r[l].astype(np.float64), out["router_logits"]) <= TOL_HIDDEN, l
        for b in range(cfg.batch):
            if set(sel[l, b].tolist()) != set(out["sel"][b].tolist()):
                srt = np.sort(out["router_logits"][b])[::-1]
                err = float(np.max(np.abs(r[l, b] - out["router_logits"][b])))
                assert srt[cfg.top_k - 1] - srt[cfg.top_k] < 2 * err, (l, b)
    refs = np.stack([model.lm_head(hid[2 * cfg.n_layers, b]) for b in range(cfg.batch)])
    assert float(np.max(np.abs(lg[:cfg.batch] - refs))) <= TOL_LOGITS_ABS
    assert all(top1_agree(lg[:cfg.batch], refs))
