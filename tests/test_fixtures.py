"""The seeded input generator: determinism, slicing and the shape of its draws."""
import numpy as np

import fixtures as fx


def test_slices_regenerate_identically():
    t = fx.tid(fx.WQ, 3)
    full = fx.normal_bf16(7, t, 10000, 0.02)
    part = fx.normal_bf16(7, t, 1000, 0.02, offset=4321)
    assert np.array_equal(full[4321:5321], part)
    assert not np.array_equal(full, fx.normal_bf16(8, t, 10000, 0.02))
    assert not np.array_equal(full, fx.normal_bf16(7, fx.tid(fx.WQ, 4), 10000, 0.02))


def test_normal_moments_and_bounds():
    x = fx.bf16_to_f32(fx.normal_bf16(0, 99, 1 << 20, 0.02)).astype(np.float64)
    assert abs(x.mean()) < 1e-4 and abs(x.std() - 0.02) < 2e-4
    assert np.abs(x).max() <= 0.02 * 2 * np.sqrt(3) * 1.01
    # fourth moment of Irwin-Hall(4) standardised: 3 - 6/(5*4) = 2.7
    z = x / x.std()
    assert abs(np.mean(z ** 4) - 2.7) < 0.05


def test_uniform_ints_range_and_spread():
    v = fx.uniform_ints(0, 5, 200000, 256, 4096)
    assert v.min() >= 256 and v.max() <= 4096
    assert abs(v.mean() - (256 + 4096) / 2) < 20
    t = fx.tokens(fx.CONFIGS["dense-8b"])
    assert t.shape == (128, 1) and t.min() >= 0 and t.max() < 128256


def test_kv_prefill_layout_and_poison():
    cfg = fx.CONFIGS["tiny"].replace(batch=2, ctx=0, ctx_lo=3, ctx_hi=9)
    S = fx.context_lengths(cfg)
    k = fx.kv_prefill(cfg, 1, 0, S, poison=True)
    for b in range(2):
        assert (k[b, :, S[b]:] == fx.BF16_NAN).all() and (k[b, :, :S[b]] != fx.BF16_NAN).all()
    idx = ((1 * cfg.n_kv_heads + 1) * cfg.max_ctx + 2) * cfg.head_dim
    ref = fx.normal_bf16(0, fx.tid(fx.K_CACHE, 1), cfg.head_dim, 1.0, offset=idx)
    assert np.array_equal(k[1, 1, 2], ref)


def test_weight_bytes_of_named_configs():
    c = fx.CONFIGS["dense-8b"]
    assert c.max_ctx == 4224
    assert abs(c.weight_bytes() / 1e9 - 16.06) < 0.01
    assert abs(fx.CONFIGS["moe-128x8"].weight_bytes() / 1e9 - 61.06) < 0.05
