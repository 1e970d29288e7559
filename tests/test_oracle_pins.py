"""Pins of the CPU oracle against things other than itself.

The pages print no worked example for the decode step (ForgeMegakernel,
arXiv 2609.12379, abstract: only the operations and the mid-state oracle idea
are named), so every pin here is a closed form, an invariant, a library
routine (PyTorch fp64) or brute force on a tiny input.  Each is chosen so that a
plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a wrong tie rule) fails at least one of them; the planted
mistakes in test_oracle_mutants.py show that.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import fixtures as fx
import oracle as ora
from tests import ref_torch
from tests.helpers import bf16_f64, expert_loader, host_caches, host_model, rel_l2

RNG = np.random.default_rng(1234)


def rand_bf16(shape, sigma=1.0):
    x = torch.from_numpy(RNG.normal(0, sigma, size=shape)).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ bfloat16 rounding

def test_bf16_roundtrip_exact():
    # every finite bf16 value widens and narrows back to itself
    hs = np.arange(0, 1 << 16, dtype=np.uint32)
    for h in hs[::97]:
        if (h & 0x7F80) == 0x7F80:
            continue
        assert ora.double_to_bf16(ora.bf16_to_double(int(h))) == int(h)


def test_bf16_ties_to_even_and_nearest():
    one = 0x3F80
    ulp = 2.0 ** -7
    assert ora.double_to_bf16(1.0 + ulp / 2) == one                   # tie -> even (down)
    assert ora.double_to_bf16(1.0 + 3 * ulp / 2) == one + 2           # tie -> even (up)
    assert ora.double_to_bf16(1.0 + ulp / 2 + 1e-12) == one + 1       # just above the tie
    assert ora.double_to_bf16(-(1.0 + ulp / 2 + 1e-12)) == 0x8000 | (one + 1)
    assert ora.double_to_bf16(0.0) == 0 and ora.double_to_bf16(-0.0) == 0x8000
    assert ora.double_to_bf16(1e300) == 0x7F80


def test_bf16_nearest_bruteforce():
    # for random doubles the result is a nearest bf16 (checked against both neighbours)
    xs = RNG.normal(0, 10, size=3000) * np.exp(RNG.uniform(-30, 30, size=3000))
    for x in xs:
        h = ora.double_to_bf16(x)
        r = ora.bf16_to_double(h)
        for nb in (h - 1, h + 1):
            rn = ora.bf16_to_double(nb & 0xFFFF)
            if math.isfinite(rn) and (nb & 0x7FFF) != 0:
                assert abs(x - r) <= abs(x - rn) + 0.0


# ------------------------------------------------------------------ RMSNorm

def test_rmsnorm_unit_rms_before_gain():
    x = RNG.normal(0, 3, size=512)
    ones = np.full(512, fx.BF16_ONE, dtype=np.uint16)
    y = ora.rmsnorm(x, ones, 0.0)
    assert abs(math.sqrt(np.mean(y * y)) - 1.0) < 1e-14


def test_rmsnorm_matches_torch():
    x = RNG.normal(0, 3, size=(1, 300))
    g = rand_bf16(300)
    y = ora.rmsnorm(x[0], g, 1e-6)
    ref = F.rms_norm(torch.from_numpy(x), (300,), torch.from_numpy(bf16_f64(g)), eps=1e-6).numpy()[0]
    assert np.max(np.abs(y - ref)) < 1e-12


# ------------------------------------------------------------------ RoPE

@pytest.mark.parametrize("d,theta", [(64, 1e4), (128, 5e5)])
def test_rope_properties(d, theta):
    v = RNG.normal(size=d)
    assert np.array_equal(ora.rope(v, 0, theta), v)                       # position 0 is the identity
    r = ora.rope(v, 777, theta)
    h = d // 2
    assert np.allclose(np.hypot(r[:h], r[h:]), np.hypot(v[:h], v[h:]), rtol=0, atol=1e-12)   # per-pair norm
    q, k = RNG.normal(size=d), RNG.normal(size=d)
    a = ora.rope(q, 1000, theta) @ ora.rope(k, 990, theta)
    b = ora.rope(q, 10, theta) @ ora.rope(k, 0, theta)
    assert abs(a - b) < 1e-9                                                 # depends only on p - p'


@pytest.mark.parametrize("d,theta", [(64, 1e4), (128, 5e5), (8, 10.0)])
def test_rope_matches_complex_form(d, theta):
    v = RNG.normal(size=d)
    for pos in (1, 5, 4223):
        ref = ref_torch.rope_complex(torch.from_numpy(v), pos, theta).numpy()
        assert np.max(np.abs(ora.rope(v, pos, theta) - ref)) < 1e-12


def test_rope_two_dim_closed_form():
    # d = 2: the single pair is rotated by pos radians counter-clockwise
    r = ora.rope(np.array([1.0, 0.0]), 3, 1e4)
    assert np.allclose(r, [math.cos(3), math.sin(3)], atol=1e-15)


# ------------------------------------------------------------------ GEMV / SwiGLU

def test_gemv_bruteforce():
    w = rand_bf16((37, 53), 0.02)
    x = RNG.normal(size=53)
    ref = np.array([sum(bf16_f64(w)[r, c] * x[c] for c in range(53)) for r in range(37)])
    assert np.max(np.abs(ora.gemv(w, x) - ref)) < 1e-13
    assert np.max(np.abs(ora.gemv(w, x) - bf16_f64(w) @ x)) < 1e-13


def test_silu_values():
    assert ora.silu(0.0) == 0.0
    for z in (-20.0, -1.5, 0.3, 2.0, 30.0):
        assert abs(ora.silu(z) - F.silu(torch.tensor(z, dtype=torch.float64)).item()) < 1e-15


def test_swiglu_matches_torch():
    H, I = 48, 80
    wg, wu, wd = rand_bf16((I, H), .1), rand_bf16((I, H), .1), rand_bf16((H, I), .1)
    x = RNG.normal(size=H)
    xt = torch.from_numpy(x)
    ref = F.linear(F.silu(F.linear(xt, torch.from_numpy(bf16_f64(wg)))) * F.linear(xt, torch.from_numpy(bf16_f64(wu))),
                   torch.from_numpy(bf16_f64(wd))).numpy()
    assert np.max(np.abs(ora.swiglu(wg, wu, wd, x) - ref)) < 1e-12


# ------------------------------------------------------------------ attention

def test_attention_single_position_returns_v():
    k, v = rand_bf16((1, 64)), rand_bf16((1, 64))
    out, p = ora.attention(RNG.normal(size=64), k, v)
    assert p[0] == 1.0 and np.array_equal(out, bf16_f64(v)[0])


def test_attention_equal_keys_gives_mean_v():
    k = np.tile(rand_bf16((1, 64)), (10, 1))
    v = rand_bf16((10, 64))
    out, p = ora.attention(RNG.normal(size=64), k, v)
    assert np.allclose(p, 0.1, atol=1e-15)
    assert np.max(np.abs(out - bf16_f64(v).mean(0))) < 1e-14


def test_attention_probs_and_sdpa():
    n, d = 300, 128
    q = RNG.normal(size=d)
    k, v = rand_bf16((n, d)), rand_bf16((n, d))
    out, p = ora.attention(q, k, v)
    assert abs(p.sum() - 1.0) < 1e-13 and (p > 0).all()
    ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None, None, None], torch.from_numpy(bf16_f64(k))[None, None],
                                         torch.from_numpy(bf16_f64(v))[None, None])[0, 0, 0].numpy()
    assert np.max(np.abs(out - ref)) < 1e-12


# ------------------------------------------------------------------ top-k routing

def test_topk_matches_torch_and_softmax_renorm():
    for _ in range(20):
        r = RNG.normal(size=128)
        sel, w = ora.topk(r, 8)
        tv, ti = torch.topk(torch.from_numpy(r), 8)
        assert np.array_equal(sel, ti.numpy())
        full = torch.softmax(torch.from_numpy(r), 0).numpy()
        assert np.allclose(w, full[sel] / full[sel].sum(), rtol=1e-13, atol=0)
        assert abs(w.sum() - 1) < 1e-14


def test_topk_ties_go_to_lower_index():
    r = np.zeros(16)
    r[[3, 9, 12]] = 2.0
    r[[5, 7]] = 1.0
    sel, w = ora.topk(r, 5)
    assert list(sel) == [3, 9, 12, 5, 7]
    sel, w = ora.topk(np.zeros(6), 6)          # all equal: identity order, uniform weights
    assert list(sel) == list(range(6)) and np.allclose(w, 1 / 6, atol=1e-16)


# ------------------------------------------------------------------ KV append, whole model

def _tiny(**kw):
    return fx.CONFIGS["tiny"].replace(**kw)


def _run_oracle(cfg, gains="ones", seed=0, steps=1):
    g, ls = host_model(cfg, seed, gains)
    S = fx.context_lengths(cfg, seed)
    kc, vc = host_caches(cfg, S, seed)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls,
                      expert_loader(cfg, seed) if cfg.n_experts else None)
    return g, ls, S, kc, vc, model


def test_kv_append_writes_only_the_new_row():
    cfg = _tiny(batch=2, ctx=0, ctx_lo=5, ctx_hi=40, steps=2)
    g, ls, S, kc, vc, model = _run_oracle(cfg)
    k0, v0 = kc.copy(), vc.copy()
    tok = fx.tokens(cfg)[0]
    model.decode_step(kc, vc, tok, S, S)
    for l in range(cfg.n_layers):
        for b in range(cfg.batch):
            mask = np.ones(cfg.max_ctx, bool)
            mask[S[b]] = False
            assert np.array_equal(kc[l, b][:, mask], k0[l, b][:, mask])
            assert np.array_equal(vc[l, b][:, mask], v0[l, b][:, mask])
            assert not np.array_equal(kc[l, b][:, S[b]], k0[l, b][:, S[b]])


def test_new_row_is_bf16_of_projected_value():
    # position 0, empty cache: attention returns exactly the new V row, and the new K row
    # is bf16 of the projected key (RoPE at position 0 is the identity)
    cfg = _tiny(ctx=0, steps=1, batch=1)
    g, ls, S, kc, vc, model = _run_oracle(cfg)
    tok = fx.tokens(cfg)[0]
    out = model.decode_step(kc, vc, tok, S, S)
    W = ls[0]
    x = bf16_f64(g["embed"])[tok[0]]
    xn = ora.rmsnorm(x, W["attn_norm"], cfg.rms_eps)
    k = bf16_f64(W["wk"]) @ xn
    v = bf16_f64(W["wv"]) @ xn
    kb = np.array([ora.double_to_bf16(t) for t in k], dtype=np.uint16).reshape(cfg.n_kv_heads, cfg.head_dim)
    vb = np.array([ora.double_to_bf16(t) for t in v], dtype=np.uint16).reshape(cfg.n_kv_heads, cfg.head_dim)
    assert np.array_equal(kc[0, 0, :, 0], kb) and np.array_equal(vc[0, 0, :, 0], vb)
    g_ = cfg.n_q_heads // cfg.n_kv_heads
    attn = np.concatenate([bf16_f64(vb[h // g_]) for h in range(cfg.n_q_heads)])
    h_attn = x + bf16_f64(W["wo"]) @ attn
    assert np.max(np.abs(out["h_attn"][0, 0] - h_attn)) < 1e-12


@pytest.mark.parametrize("name,gains,kw", [
    ("tiny", "ones", {}),
    ("tiny", "random", {"batch": 3, "ctx": 0, "ctx_lo": 0, "ctx_hi": 60, "steps": 4}),
    ("tiny", "random", {"qk_norm": True, "tied_embeddings": True, "rope_theta": 5e5}),
])
def test_whole_step_matches_torch_reference(name, gains, kw):
    cfg = fx.CONFIGS[name].replace(**kw)
    g, ls, S, kc, vc, model = _run_oracle(cfg, gains)
    kc2, vc2 = kc.copy(), vc.copy()
    tok = fx.tokens(cfg)[0]
    pos = S.copy()
    out = model.decode_step(kc, vc, tok, pos, S)
    ref = ref_torch.decode_step(cfg, g, ls, kc2, vc2, tok, pos, S)
    # the only rounding that both sides take is the bf16 narrowing of the appended K/V rows
    diff = np.count_nonzero(kc != kc2) + np.count_nonzero(vc != vc2)
    assert diff <= 2
    tol = 1e-9 if diff == 0 else 1e-3
    for key in ("h_attn", "h_mlp"):
        assert rel_l2(out[key], ref[key]) < tol, key
    assert rel_l2(out["logits"], ref["logits"]) < tol


def test_moe_step_matches_torch_reference():
    cfg = fx.ModelConfig("tiny-moe", n_layers=2, hidden=128, n_q_heads=4, n_kv_heads=2, head_dim=32, ffn_dim=0,
                         vocab=256, n_experts=8, top_k=3, expert_ffn_dim=48, batch=2, ctx_lo=3, ctx_hi=30, steps=2)
    g, ls, S, kc, vc, model = _run_oracle(cfg, "random")
    kc2, vc2 = kc.copy(), vc.copy()
    tok = fx.tokens(cfg)[0]
    out = model.decode_step(kc, vc, tok, S, S)
    ref = ref_torch.decode_step(cfg, g, ls, kc2, vc2, tok, S, S, expert_fn=expert_loader(cfg))
    assert np.array_equal(out["sel"], ref["sel"])
    assert np.max(np.abs(out["sel_w"] - ref["sel_w"])) < 1e-12
    for key in ("h_attn", "h_mlp", "router_logits", "logits"):
        assert rel_l2(out[key], ref[key]) < 1e-9, key


def _moe_cfg(E, k):
    return fx.ModelConfig("moe-pin", n_layers=1, hidden=64, n_q_heads=2, n_kv_heads=1, head_dim=32, ffn_dim=0,
                          vocab=64, n_experts=E, top_k=k, expert_ffn_dim=40, batch=1, ctx=4, steps=1)


def test_moe_uniform_router_all_experts_is_mean():
    cfg = _moe_cfg(6, 6)
    g, ls, S, kc, vc, model = _run_oracle(cfg, "random")
    ls[0]["router"][:] = 0                                     # uniform router
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls, expert_loader(cfg))
    tok = fx.tokens(cfg)[0]
    out = model.decode_step(kc, vc, tok, S, S)
    h = out["h_attn"][0, 0]
    xn = ora.rmsnorm(h, ls[0]["mlp_norm"], cfg.rms_eps)
    ys = [ora.swiglu(*[expert_loader(cfg)(0, e)[n] for n in ("w_gate", "w_up", "w_down")], xn) for e in range(6)]
    assert np.max(np.abs(out["h_mlp"][0, 0] - (h + np.mean(ys, axis=0)))) < 1e-12
    assert list(out["sel"][0, 0]) == list(range(6))


def test_moe_one_hot_router_top1_is_dense_swiglu():
    cfg = _moe_cfg(5, 1)
    g, ls, S, kc, vc, model = _run_oracle(cfg, "random")
    # a router whose row 3 is the only non-zero one: token with positive projection picks expert 3
    ls[0]["router"][:] = 0
    ls[0]["router"][3] = ls[0]["mlp_norm"]                     # logit_3 = xn . g  = sum g_i^2 x_i/rms
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls, expert_loader(cfg))
    tok = fx.tokens(cfg)[0]
    out = model.decode_step(kc, vc, tok, S, S)
    h = out["h_attn"][0, 0]
    xn = ora.rmsnorm(h, ls[0]["mlp_norm"], cfg.rms_eps)
    e = 3 if out["router_logits"][0, 0, 3] > 0 else 0
    assert out["sel"][0, 0, 0] == e and out["sel_w"][0, 0, 0] == 1.0
    y = ora.swiglu(*[expert_loader(cfg)(0, e)[n] for n in ("w_gate", "w_up", "w_down")], xn)
    assert np.max(np.abs(out["h_mlp"][0, 0] - (h + y))) < 1e-12


def test_step_rejects_out_of_range():
    cfg = _tiny(steps=1)
    g, ls, S, kc, vc, model = _run_oracle(cfg)
    with pytest.raises(ValueError):
        model.decode_step(kc, vc, [0], [cfg.max_ctx], [cfg.max_ctx])


# ------------------------------------------------------------------ low-bit weights (fp8 / nvfp4)

def _e4m3_torch(codes):
    """E4M3 codes decoded by PyTorch's float8_e4m3fn (a library routine)."""
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = _e4m3_torch(codes)
    got = np.array([ora.e4m3_to_double(int(c)) for c in codes])
    assert np.array_equal(np.isnan(got), np.isnan(ref)) and np.isnan(got).sum() == 2  # 0x7F, 0xFF
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def test_e4m3_closed_forms():
    assert ora.e4m3_to_double(0x38) == 1.0                 # exponent 7 = bias
    assert ora.e4m3_to_double(0x7E) == 448.0               # largest finite: 2^8 * 1.75
    assert ora.e4m3_to_double(0x01) == 2.0 ** -9           # smallest subnormal
    assert ora.e4m3_to_double(0x07) == 7 * 2.0 ** -9       # largest subnormal
    assert ora.e4m3_to_double(0x08) == 2.0 ** -6           # smallest normal
    assert ora.e4m3_to_double(0xC0) == -2.0


def test_e2m1_every_code():
    # the OCP 4-bit floating-point format's magnitudes; bit 3 is the sign
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for n in range(16):
        v = ora.e2m1_to_double(n)
        assert abs(v) == mags[n & 7] and (math.copysign(1.0, v) < 0) == bool(n & 8)


def test_gemv_fp8_matches_dequantized_torch():
    rows, cols, block = 7, 300, 128                        # a ragged last block of 44 columns
    w = RNG.integers(0, 256, size=(rows, cols)).astype(np.uint8)
    w[(w & 0x7F) == 0x7F] = 0x3C                           # no NaN codes
    nb = (cols + block - 1) // block
    scale = RNG.uniform(0.01, 2.0, size=(rows, nb)).astype(np.float32)
    x = RNG.normal(0, 1, size=cols)
    wd = _e4m3_torch(w.reshape(-1)).reshape(rows, cols) * np.repeat(scale.astype(np.float64), block, axis=1)[:, :cols]
    ref = (torch.from_numpy(wd) @ torch.from_numpy(x)).numpy()
    y = ora.gemv_fp8(w, scale, block, x)
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_gemv_nvfp4_nibble_order_and_scales():
    # one row: byte 0x21 holds column 0 = 0.5 (low nibble 1) and column 1 = 1.0 (high nibble 2)
    w = np.zeros((1, 8), dtype=np.uint8)
    w[0, 0] = 0x21
    scale = np.array([[0x40]], dtype=np.uint8)             # E4M3 0x40 = 2.0, for columns 0..15
    x = np.zeros(16)
    x[0], x[1] = 3.0, 5.0
    y = ora.gemv_nvfp4(w, scale, 0.25, x)
    assert y[0] == (0.5 * 3.0 + 1.0 * 5.0) * 2.0 * 0.25


def test_gemv_nvfp4_matches_dequantized():
    rows, cols = 5, 64
    nib = RNG.integers(0, 16, size=(rows, cols)).astype(np.uint8)
    w = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    sc = RNG.integers(0x20, 0x50, size=(rows, cols // 16)).astype(np.uint8)   # finite E4M3 scales
    ts = 0.0625
    x = RNG.normal(0, 1, size=cols)
    table = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    vals = np.where(nib & 8, -1.0, 1.0) * table[nib & 7]
    wd = vals * np.repeat(_e4m3_torch(sc.reshape(-1)).reshape(rows, -1), 16, axis=1) * ts
    ref = wd @ x
    y = ora.gemv_nvfp4(w, sc, ts, x)
    assert np.max(np.abs(y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_fp8_step_equals_bf16_step_when_the_weights_agree():
    # fp8 projections whose E4M3 code x power-of-two block scale is exactly representable in bf16
    # (4 significant bits): the oracle's fp8 step and its bf16 step on those bf16 values must agree
    # bit for bit (same products, same summation order)
    cfg = fx.CONFIGS["tiny"].replace(ffn_dim=320)
    g, ls = host_model(cfg, gains="random")
    block = 128
    gen = torch.Generator().manual_seed(7)
    for lw in ls:
        for name in ora.FP8_MATRICES:
            rows, cols = lw[name].shape
            codes = (torch.randn(rows, cols, generator=gen, dtype=torch.float32) * 8).to(torch.float8_e4m3fn)
            nb = (cols + block - 1) // block
            k = torch.randint(-10, -6, (rows, nb), generator=gen)
            scale = torch.pow(2.0, k.to(torch.float64)).to(torch.float32)
            w = codes.to(torch.float64) * scale.to(torch.float64).repeat_interleave(block, dim=1)[:, :cols]
            wb = w.to(torch.bfloat16)
            assert torch.equal(wb.to(torch.float64), w)          # exact in bf16
            lw[name] = wb.view(torch.int16).numpy().view(np.uint16)
            lw[name + "_fp8"] = (codes.view(torch.uint8).numpy(), scale.numpy())
    S = fx.context_lengths(cfg)
    outs = []
    for fp8 in (0, block):
        kc, vc = host_caches(cfg, S)
        model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls, fp8_block=fp8)
        outs.append((model.decode_step(kc, vc, fx.tokens(cfg)[0], S, S), kc, vc))
    (a, ka, va), (b, kb, vb) = outs
    for key in ("h_attn", "h_mlp", "logits"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(ka, kb) and np.array_equal(va, vb)


def test_fp8_step_uses_the_fp8_weights():
    # the same model with its fp8 codes perturbed (bf16 matrices unchanged) must change the fp8 step only
    cfg = fx.CONFIGS["tiny"].replace(ffn_dim=320, n_layers=1)
    g, ls = host_model(cfg)
    gen = torch.Generator().manual_seed(3)
    for lw in ls:
        for name in ora.FP8_MATRICES:
            rows, cols = lw[name].shape
            codes = (torch.randn(rows, cols, generator=gen) * 8).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            lw[name + "_fp8"] = (codes, np.full((rows, (cols + 127) // 128), 2.0 ** -8, dtype=np.float32))
    S = fx.context_lengths(cfg)
    res = []
    for bump in (False, True):
        if bump:
            c, s = ls[0]["wo_fp8"]
            c = c.copy()
            c[0, 0] ^= 0x08                                     # one code of o_proj
            ls[0]["wo_fp8"] = (c, s)
        kc, vc = host_caches(cfg, S)
        m = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls, fp8_block=128)
        res.append(m.decode_step(kc, vc, fx.tokens(cfg)[0], S, S)["h_attn"])
    d = np.abs(res[1] - res[0]).reshape(-1)
    assert d[0] > 0 and np.count_nonzero(d) == 1                # o_proj row 0 only


def test_fp8_step_refuses_a_mixture_of_experts_model():
    # fp8 forms exist for wq wk wv wo and the dense gate / up / down only: a MoE model asked to run
    # in fp8 is refused on both sides of the binding instead of silently running its experts in bf16
    cfg = fx.CONFIGS["tiny"].replace(ffn_dim=0, n_experts=4, top_k=2, expert_ffn_dim=64, n_layers=1)
    g, ls = host_model(cfg)
    with pytest.raises(ValueError):
        ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls, expert_loader(cfg), fp8_block=128)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls, expert_loader(cfg))
    model.m.d.fp8_block = 128                                   # the C entry point's own check
    kc, vc = host_caches(cfg, fx.context_lengths(cfg))
    S = fx.context_lengths(cfg)
    with pytest.raises(ValueError):
        model.layer_forward(0, np.zeros((cfg.batch, cfg.hidden)), kc[0], vc[0], S, S)
