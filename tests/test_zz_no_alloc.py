"""mk_decode_step_noalloc against the handle-based mk_decode_step, on the GPU, through the C ABI.

The entry point exists for callers that cannot call cudaMalloc where they
decode (a plugin inside an engine that owns all device memory, a real-time
path that must not enter the allocator): its state lives in one static 8 MiB
device array.  It runs the same kernel on the same instruction lists as the
allocating path, with fixed-order reductions, so two calls in a row must give
bit-identical logits and appended K/V rows.  This file is collected last on
purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import fixtures as fx
from fixtures.device import device_caches, device_model
from tests.gpu_harness import bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("dense-0.6b", {}),
                                     ("tiny", {"batch": 4, "ffn_dim": 704, "ctx": 0, "ctx_lo": 5, "ctx_hi": 130})])
def test_noalloc_matches_allocating_path_two_calls(name, kw):
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS[name].replace(**kw)
    S0 = fx.context_lengths(cfg)
    toks = fx.tokens(cfg)
    w = device_model(cfg)
    kc_a, vc_a = device_caches(cfg, S0)
    kc_b, vc_b = kc_a.clone(), vc_a.clone()
    dec = mk.Decoder(cfg, w, kc_a, vc_a)
    desc, wst, kv, keep = mk.weight_structs(cfg, w, kc_b, vc_b)
    la = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    lb = torch.full_like(la, float("nan"))
    stream = torch.cuda.current_stream()
    for t in range(2):
        S = (S0 + t).astype(np.int32)
        d_tok = torch.from_numpy(toks[t].copy()).cuda()
        d_len = torch.from_numpy(S).cuda()
        dec.step(d_tok, d_len, d_len, la)
        assert dec.status() == mk.MK_OK
        rc = mk.mk_decode_step_noalloc(ctypes.byref(desc), ctypes.byref(wst), ctypes.byref(kv), d_tok.data_ptr(),
                                       d_len.data_ptr(), d_len.data_ptr(), stream.cuda_stream, lb.data_ptr())
        assert rc == mk.MK_OK, mk.mk_status_string(rc)
        torch.cuda.synchronize()
        a, b = la.cpu().numpy(), lb.cpu().numpy()
        assert np.isfinite(b).all()
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), t
        for cache_a, cache_b in ((kc_a, kc_b), (vc_a, vc_b)):
            for b in range(cfg.batch):
                ra = bits(cache_a[:, b, :, S[b]].contiguous())
                rb = bits(cache_b[:, b, :, S[b]].contiguous())
                assert np.array_equal(ra, rb), (t, b)
        lb.fill_(float("nan"))
    dec.close()
    del keep


def test_noalloc_rejects_state_beyond_the_static_array():
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"]
    w = device_model(cfg)
    big = cfg.replace(ctx=300000 - cfg.steps)            # RoPE table alone would need ~77 MB
    kc, vc = device_caches(big, seq_lens=[0])            # caches of the full shape, so no launch could overrun
    desc, wst, kv, keep = mk.weight_structs(big, w, kc, vc)
    d = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    rc = mk.mk_decode_step_noalloc(ctypes.byref(desc), ctypes.byref(wst), ctypes.byref(kv), d.data_ptr(),
                                   d.data_ptr(), d.data_ptr(), torch.cuda.current_stream().cuda_stream,
                                   out.data_ptr())
    assert rc == mk.MK_ERR_UNSUPPORTED
