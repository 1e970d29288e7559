"""Failure detection on the GPU without a GPU fault.

Faults are made on the host: a lowering with one dependency no instruction
can satisfy (MK_FAULT_INJECT=wait) and out-of-range per-step inputs.  Every
in-kernel wait is bounded, so the step ends with a device status the host
reads, and the handle (and the GPU) stays usable.
"""
import numpy as np
import pytest
import torch

import fixtures as fx
from fixtures.device import device_caches, device_model
from tests.gpu_harness import assert_parity, bits, run_teacher_forced

pytestmark = pytest.mark.gpu


def _inputs(cfg):
    S0 = fx.context_lengths(cfg)
    return S0, device_model(cfg), device_caches(cfg, S0)


def test_unsatisfiable_wait_times_out_and_recovers(monkeypatch):
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"]
    S0, w, (kc, vc) = _inputs(cfg)
    monkeypatch.setenv("MK_FAULT_INJECT", "wait")
    dec = mk.Decoder(cfg, w, kc, vc, wait_timeout_ns=20_000_000)   # 20 ms bound on every wait
    monkeypatch.delenv("MK_FAULT_INJECT")
    tok = torch.from_numpy(fx.tokens(cfg)[0].copy()).cuda()
    sl = torch.from_numpy(S0.copy()).cuda()
    logits = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    dec.step(tok, sl, sl, logits)
    assert dec.status() == mk.MK_ERR_DEVICE_TIMEOUT
    assert dec.status() == mk.MK_OK                       # read once, then cleared
    dec.step(tok, sl, sl, logits)                         # the same plan fails the same way, cleanly
    assert dec.status() == mk.MK_ERR_DEVICE_TIMEOUT
    dec.close()
    torch.cuda.synchronize()
    assert_parity(run_teacher_forced(cfg, steps=2))       # the GPU and the library are fine


def test_out_of_range_inputs_are_rejected_before_any_work():
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"]
    S0, w, (kc, vc) = _inputs(cfg)
    dec = mk.Decoder(cfg, w, kc, vc)
    logits = torch.zeros((1, cfg.vocab), dtype=torch.float32, device="cuda")
    k0, v0 = bits(kc).copy(), bits(vc).copy()
    tok = torch.from_numpy(fx.tokens(cfg)[0].copy()).cuda()
    for lens, toks in (([cfg.max_ctx], tok), ([-1], tok), ([int(S0[0])], torch.tensor([cfg.vocab], dtype=torch.int32).cuda())):
        sl = torch.tensor(lens, dtype=torch.int32).cuda()
        dec.step(toks, sl, sl, logits)
        assert dec.status() == mk.MK_ERR_RANGE
        assert np.array_equal(bits(kc), k0) and np.array_equal(bits(vc), v0)
        assert float(logits.abs().max()) == 0.0
    sl = torch.from_numpy(S0.copy()).cuda()
    dec.step(tok, sl, sl, logits)
    assert dec.status() == mk.MK_OK and float(logits.abs().max()) > 0
    dec.close()


def test_create_rejects_bad_descriptors():
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"]
    S0, w, (kc, vc) = _inputs(cfg)
    with pytest.raises(mk.MkError):
        mk.Decoder(cfg.replace(head_dim=96), w, kc, vc)
    misaligned = dict(w)
    misaligned["embed"] = w["embed"].view(-1)[1:]          # 2-byte offset
    with pytest.raises(mk.MkError):
        mk.Decoder(cfg, misaligned, kc, vc)
