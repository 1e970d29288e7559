"""The trace helpers on a synthetic timeline (no GPU): what each reported phase measures."""
import numpy as np

import auto_regressive_decode_b200.mk as mk
import fixtures as fx
from auto_regressive_decode_b200.trace import format_breakdown, handoff_costs, layer_breakdown, summarize


def synthetic(plan):
    """Stamps (ns) from each instruction's op and layer: ready at 100 us per layer + 10 us per op,
    then prologue 1, first stage 2, stream 3, epilogue 4 us; start 0.5 us before ready;
    producer's copies 0.25 us after start and 0.25 us before done."""
    ops = plan.instrs[:, 0] & 0xFF
    layers = plan.instrs[:, 0] >> 8
    ready = (100_000 * (layers + 1) + 10_000 * ops).astype(np.int64)
    t = np.zeros((len(ops), 8), dtype=np.int64)
    t[:, 1] = ready
    t[:, 4] = ready + 1000
    t[:, 5] = ready + 3000
    t[:, 6] = ready + 6000
    t[:, 2] = ready + 10_000
    t[:, 0] = ready - 500
    t[:, 3] = t[:, 0] + 250
    t[:, 7] = t[:, 2] - 250
    return t


def test_layer_breakdown_phases():
    cfg = fx.CONFIGS["tiny"]
    plan = mk.Plan(mk.model_desc(cfg), 4)
    t = synthetic(plan)
    rows = {r["op"]: r for r in layer_breakdown(plan, t, 1)}
    assert set(rows) == {"qkv", "attn", "oproj", "gateup", "down"}
    # layer 0's last done: its down (op 6) at 100 + 60 + 10 us
    prev = 100 + 60 + 10
    for name, op in (("qkv", 2), ("attn", 3), ("oproj", 4), ("gateup", 5), ("down", 6)):
        r = rows[name]
        ready = 200 + 10 * op - prev
        assert abs(r["ready"] - ready) < 1e-9
        assert abs(r["prologue"] - 1) < 1e-9 and abs(r["first_stage"] - 2) < 1e-9
        assert abs(r["stream"] - 3) < 1e-9 and abs(r["epilogue"] - 4) < 1e-9
        assert abs(r["done"] - (ready + 10)) < 1e-9 and abs(r["done_max"] - (ready + 10)) < 1e-9
        assert abs(r["producer_first"] - (ready - 0.25)) < 1e-9
        assert abs(r["producer_last"] - (ready + 9.75)) < 1e-9
    assert "stream" in format_breakdown(list(rows.values()))
    assert "layer 0" in summarize(plan, t)


def test_handoff_costs_same_sm_only():
    cfg = fx.CONFIGS["tiny"]
    plan = mk.Plan(mk.model_desc(cfg), 4)
    t = synthetic(plan)
    h = handoff_costs(plan, t)
    # on an SM, qkv (op 2) is followed by attention of the same layer: start = ready(attn) - 0.5,
    # done(qkv) = ready(qkv) + 10, ready(attn) - ready(qkv) = 10 us -> hand-off -0.5 us
    assert abs(h["qkv"] - (-0.5)) < 1e-9
    assert "lmhead" not in h  # an SM's last instruction has no successor
