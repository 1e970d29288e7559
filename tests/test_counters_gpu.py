"""Per-step audit of the dependency counters, read back on the host.

Every instruction that raises a counter does so once per step, so after k
steps each counter holds exactly k times its per-step target (the number of
its producers in the lowering); an extra, lost or repeated bump shows up here
even when the outputs happen to be right.  A failing step's status read
clears the counters and restarts the count.
"""
import numpy as np
import pytest
import torch

import fixtures as fx
from fixtures.device import device_caches, device_model

pytestmark = pytest.mark.gpu


def _decoder(cfg, **kw):
    import auto_regressive_decode_b200.mk as mk
    S0 = fx.context_lengths(cfg)
    w = device_model(cfg)
    kc, vc = device_caches(cfg, S0)
    dec = mk.Decoder(cfg, w, kc, vc, **kw)
    plan = mk.Plan(mk.model_desc(cfg), torch.cuda.get_device_properties(0).multi_processor_count)
    return dec, plan, S0, (w, kc, vc)


def _step(dec, cfg, S0, t, logits):
    S = torch.from_numpy((S0 + t).astype(np.int32)).cuda()
    dec.step(torch.from_numpy(fx.tokens(cfg)[t].copy()).cuda(), S, S, logits)


@pytest.mark.parametrize("kw", [{}, {"batch": 4, "ffn_dim": 704, "ctx": 0, "ctx_lo": 5, "ctx_hi": 130},
                                {"n_experts": 8, "top_k": 2, "expert_ffn_dim": 128, "batch": 2}])
def test_each_counter_counts_its_producers_every_step(kw):
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"].replace(**kw)
    dec, plan, S0, keep = _decoder(cfg)
    target = plan.targets.astype(np.uint32)
    assert (target > 0).sum() > 0
    logits = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    assert np.array_equal(dec.counters(), np.zeros_like(target))
    for t in range(3):
        _step(dec, cfg, S0, t, logits)
        assert dec.status() == mk.MK_OK
        got = dec.counters()
        bad = np.nonzero(got != (t + 1) * target)[0]
        assert bad.size == 0, (t, bad[:8], got[bad[:8]], target[bad[:8]])
    dec.close()


def test_a_failed_step_restarts_the_count(monkeypatch):
    import auto_regressive_decode_b200.mk as mk
    cfg = fx.CONFIGS["tiny"]
    monkeypatch.setenv("MK_FAULT_INJECT", "wait")
    dec, plan, S0, keep = _decoder(cfg, wait_timeout_ns=20_000_000)
    monkeypatch.delenv("MK_FAULT_INJECT")
    logits = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    _step(dec, cfg, S0, 0, logits)
    assert dec.status() == mk.MK_ERR_DEVICE_TIMEOUT                 # the read clears the counters
    assert not dec.counters().any()
    dec.close()
    dec, plan, S0, keep = _decoder(cfg)                              # the normal lowering counts again
    _step(dec, cfg, S0, 0, logits)
    assert dec.status() == mk.MK_OK
    assert np.array_equal(dec.counters(), plan.targets.astype(np.uint32))
    dec.close()
