"""On-device greedy decoding (mk_decode_greedy) on the GPU, through the C ABI.

The loop feeds each step's arg-max back as the next token without the host.
Checks: (1) each picked token is the arg-max of that step's GPU logits (largest
logit, ties to the lowest id), bit-exact, as recomputed by replaying the picked
tokens teacher-forced through mk_decode_step; (2) the replay leaves the KV
caches bit-identical to the loop's (the same kernel on the same inputs);
(3) every pick is the oracle's arg-max (batch-1 CUDA-core kernel) or an oracle
top-1 token up to the tie margin of the parity harness (tensor-core kernel),
the oracle run on the same (picked) tokens; (4) a loop that runs a
sequence past max_ctx reports MK_ERR_RANGE and the handle recovers.
"""
import numpy as np
import pytest
import torch

import fixtures as fx
import oracle as ora
from fixtures.device import device_caches, device_model
from tests.gpu_harness import bits, tensor_core_kernel, top1_agree, top1_exact
from tests.helpers import expert_loader, host_caches, host_model

pytestmark = pytest.mark.gpu


def first_argmax(x):
    """Largest value, ties to the lowest index (numpy's argmax already keeps the first)."""
    return int(np.argmax(x))


@pytest.mark.parametrize("name,kw,steps", [
    ("tiny", {}, 12),
    ("tiny", {"batch": 4, "ffn_dim": 704, "ctx": 0, "ctx_lo": 5, "ctx_hi": 100}, 8),
    ("tiny", {"ffn_dim": 0, "n_experts": 8, "top_k": 2, "expert_ffn_dim": 128, "batch": 3, "ctx": 0, "ctx_lo": 2,
              "ctx_hi": 90}, 6),
])
def test_greedy_loop_matches_replay_and_oracle(name, kw, steps):
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS[name].replace(**kw)
    S0 = fx.context_lengths(cfg)
    x0 = fx.tokens(cfg)[0]
    w = device_model(cfg, gains="random")
    kc, vc = device_caches(cfg, S0)
    k_rep, v_rep = kc.clone(), vc.clone()
    dec = mk.Decoder(cfg, w, kc, vc)
    d_tok = torch.from_numpy(x0.copy()).cuda()
    d_len = torch.from_numpy(S0.copy()).cuda()
    picks = torch.full((steps, cfg.batch), -1, dtype=torch.int32, device="cuda")
    last = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    dec.greedy(steps, d_tok, d_len, picks, last)
    torch.cuda.synchronize()
    assert dec.status() == mk.MK_OK
    picks = picks.cpu().numpy()
    assert (d_len.cpu().numpy() == S0).all() and (d_tok.cpu().numpy() == x0).all()   # inputs only read
    dec.close()

    # replay teacher-forced on the picked tokens; oracle on the same tokens
    rep = mk.Decoder(cfg, w, k_rep, v_rep)
    g, ls = host_model(cfg, gains="random")
    okc, ovc = host_caches(cfg, S0)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls,
                      expert_loader(cfg) if cfg.n_experts else None)
    logits = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    tok = x0.copy()
    agree = []
    for t in range(steps):
        S = (S0 + t).astype(np.int32)
        ds = torch.from_numpy(S.copy()).cuda()
        rep.step(torch.from_numpy(tok.copy()).cuda(), ds, ds, logits)
        lg = logits.cpu().numpy()
        for b in range(cfg.batch):
            assert picks[t, b] == first_argmax(lg[b]), (t, b)
        ref = model.decode_step(okc, ovc, tok, S, S)
        agree += (top1_agree if tensor_core_kernel(cfg) else top1_exact)(lg.astype(np.float64), ref["logits"])
        tok = picks[t].astype(np.int32)
    assert rep.status() == mk.MK_OK
    np.testing.assert_array_equal(lg, last.cpu().numpy())
    assert np.array_equal(bits(kc), bits(k_rep)) and np.array_equal(bits(vc), bits(v_rep))
    assert np.mean(agree) >= 0.99, np.mean(agree)
    rep.close()


def test_greedy_loop_past_max_ctx_is_a_range_error():
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"]
    S0 = np.array([cfg.max_ctx - 2], dtype=np.int32)       # room for two steps only
    w = device_model(cfg)
    kc, vc = device_caches(cfg, S0)
    dec = mk.Decoder(cfg, w, kc, vc)
    d_tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    d_len = torch.from_numpy(S0.copy()).cuda()
    picks = torch.zeros((4, 1), dtype=torch.int32, device="cuda")
    dec.greedy(4, d_tok, d_len, picks)
    torch.cuda.synchronize()
    assert dec.status() == mk.MK_ERR_RANGE
    dec.greedy(2, d_tok, d_len, picks)                      # recovered: two steps fit
    torch.cuda.synchronize()
    assert dec.status() == mk.MK_OK
    dec.close()
