"""Paged KV cache (block table into a page pool) on the GPU, through the C ABI.

The same model and inputs run with the contiguous cache and with a paged
pool whose pages are a seeded random permutation (spare pages poisoned with
NaN): every step's logits and hidden states must be bit-identical (the same
arithmetic, other addresses), the appended rows must land in the right
pages, and pages the block table does not reference must stay untouched.
Both kernels are covered (batch 1: CUDA-core GEMVs; batch 3 and MoE:
tensor-core kernel).  The contiguous path itself is checked against the
oracle in tests/test_parity_gpu.py.
"""
import numpy as np
import pytest
import torch

import fixtures as fx
from fixtures.device import device_caches, device_model

pytestmark = pytest.mark.gpu

NAN_BITS = 0x7FC0  # bf16 quiet NaN


def to_pool(cache, cfg, page, n_pages, table):
    """Contiguous [L][B][nkv][T][hd] -> pool [L][n_pages][nkv][page][hd] by the block table."""
    L, B, nkv, T, hd = cache.shape
    pool = torch.full((L, n_pages, nkv, page, hd), NAN_BITS, dtype=torch.int16, device=cache.device)
    c16 = cache.view(torch.int16)
    for b in range(B):
        for j in range(table.shape[1]):
            lo, hi = j * page, min(T, (j + 1) * page)
            pool[:, table[b, j], :, :hi - lo] = c16[:, b, :, lo:hi]
    return pool.view(torch.bfloat16)


def from_pool(pool, cfg, shape, page, table):
    L, B, nkv, T, hd = shape
    out = torch.empty(shape, dtype=torch.int16, device=pool.device)
    p16 = pool.view(torch.int16)
    for b in range(B):
        for j in range(table.shape[1]):
            lo, hi = j * page, min(T, (j + 1) * page)
            out[:, b, :, lo:hi] = p16[:, table[b, j], :, :hi - lo]
    return out


@pytest.mark.parametrize("kw", [
    {"n_q_heads": 4, "n_kv_heads": 2, "head_dim": 128, "ctx": 200, "steps": 3},                       # batch 1
    {"n_q_heads": 8, "n_kv_heads": 2, "head_dim": 128, "batch": 3, "ffn_dim": 704, "ctx": 0, "ctx_lo": 5,
     "ctx_hi": 260, "steps": 3},                                                                       # tensor cores
    {"n_q_heads": 4, "n_kv_heads": 2, "head_dim": 128, "batch": 2, "ffn_dim": 0, "n_experts": 8, "top_k": 2,
     "expert_ffn_dim": 128, "ctx": 0, "ctx_lo": 100, "ctx_hi": 300, "steps": 2},                      # MoE
])
def test_paged_matches_contiguous_bit_for_bit(kw):
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"].replace(**kw)
    page = 32768 // (2 * cfg.head_dim)
    stride = -(-cfg.max_ctx // page)
    n_pages = cfg.batch * stride + 5
    rng = np.random.default_rng(7)
    table = rng.permutation(n_pages)[:cfg.batch * stride].reshape(cfg.batch, stride).astype(np.int32)
    S0 = fx.context_lengths(cfg)
    toks = fx.tokens(cfg)
    w = device_model(cfg, gains="random")
    kc, vc = device_caches(cfg, S0, poison=True)
    kp, vp = to_pool(kc, cfg, page, n_pages, table), to_pool(vc, cfg, page, n_pages, table)
    kp0, vp0 = kp.clone(), vp.clone()
    d_table = torch.from_numpy(table).cuda()
    dec_c = mk.Decoder(cfg, w, kc, vc)
    dec_p = mk.Decoder(cfg, w, kp, vp, block_table=d_table, page_size=page)
    la = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    lb = torch.empty_like(la)
    for t in range(cfg.steps):
        S = torch.from_numpy((S0 + t).astype(np.int32)).cuda()
        tk = torch.from_numpy(toks[t].copy()).cuda()
        dec_c.step(tk, S, S, la)
        dec_p.step(tk, S, S, lb)
        torch.cuda.synchronize()
        assert dec_c.status() == mk.MK_OK and dec_p.status() == mk.MK_OK
        assert torch.equal(la, lb), t
        assert torch.equal(dec_c.hidden_states(), dec_p.hidden_states()), t
    # the pool, read back through the table, equals the contiguous cache (appended rows included)
    for pool, cont in ((kp, kc), (vp, vc)):
        assert torch.equal(from_pool(pool, cfg, tuple(cont.shape), page, table), cont.view(torch.int16))
    # unreferenced pages untouched
    spare = sorted(set(range(n_pages)) - set(table.ravel().tolist()))
    assert torch.equal(kp.view(torch.int16)[:, spare], kp0.view(torch.int16)[:, spare])
    assert torch.equal(vp.view(torch.int16)[:, spare], vp0.view(torch.int16)[:, spare])
    dec_c.close()
    dec_p.close()


def test_paged_page_outside_the_pool_is_a_range_error():
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"].replace(n_q_heads=4, n_kv_heads=2, head_dim=128, ctx=200, steps=1)
    page = 128
    stride = -(-cfg.max_ctx // page)
    n_pages = stride
    table = np.arange(stride, dtype=np.int32).reshape(1, stride)
    w = device_model(cfg)
    kc, vc = device_caches(cfg)
    kp, vp = to_pool(kc, cfg, page, n_pages, table), to_pool(vc, cfg, page, n_pages, table)
    d_table = torch.from_numpy(table).cuda()
    dec = mk.Decoder(cfg, w, kp, vp, block_table=d_table, page_size=page)
    S = torch.tensor([200], dtype=torch.int32, device="cuda")
    tk = torch.zeros(1, dtype=torch.int32, device="cuda")
    logits = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    d_table[0, 1] = n_pages                     # page 1 (positions 128..255) outside the pool
    dec.step(tk, S, S, logits)
    torch.cuda.synchronize()
    assert dec.status() == mk.MK_ERR_RANGE
    d_table[0, 1] = 1                           # repaired: the handle works again
    dec.step(tk, S, S, logits)
    torch.cuda.synchronize()
    assert dec.status() == mk.MK_OK
    dec.close()
