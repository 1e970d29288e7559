"""Timeline of one decode step from the kernel's per-instruction timestamps.

Create the handle with ``MK_TRACE=1`` in the environment, run a step, then::

    t = mk.decoder_trace(decoder)        # int64 [n_instr][8]
    print(summarize(plan, t))

Stamps per instruction (ns, %globaltimer): 0 consumer start, 1 dependency
satisfied, 2 compute done, 3 producer's first copy issued, 4 prologue done,
5 first stage landed, 6 last stage consumed, 7 producer's last copy issued.
"""
from __future__ import annotations

import numpy as np

from .mk import OP_NAMES


def op_table(plan, trace):
    """Per op kind: count, mean wait (start->ready) and busy (ready->done) time in us."""
    ops = plan.instrs[:, 0] & 0xFF
    t = trace.astype(np.int64)
    rows = []
    for op in sorted(set(ops.tolist())):
        m = ops == op
        wait = (t[m, 1] - t[m, 0]) / 1e3
        busy = (t[m, 2] - t[m, 1]) / 1e3
        rows.append((OP_NAMES.get(op, str(op)), int(m.sum()), float(wait.mean()), float(np.median(wait)),
                     float(busy.mean()), float(wait.sum() + busy.sum())))
    return rows


def layer_phases(plan, trace, layer):
    """For each op of one layer: first ready, last done (us from the step's first stamp)."""
    t = trace.astype(np.int64)
    t0 = t[:, 0].min()
    ops = plan.instrs[:, 0] & 0xFF
    layers = plan.instrs[:, 0] >> 8
    out = []
    for op in sorted(set(ops[layers == layer].tolist())):
        m = (ops == op) & (layers == layer)
        out.append((OP_NAMES.get(op, str(op)), float((t[m, 1].min() - t0) / 1e3), float((t[m, 1].max() - t0) / 1e3),
                    float((t[m, 2].max() - t0) / 1e3)))
    return out


def summarize(plan, trace) -> str:
    t = trace.astype(np.int64)
    span = (t[:, 2].max() - t[:, 0].min()) / 1e3
    lines = [f"step span {span:.1f} us over {plan.n_sm} SMs, {len(t)} instructions",
             f"{'op':>10} {'count':>6} {'wait_mean':>10} {'wait_med':>9} {'busy_mean':>10} {'sm_us_total':>12}"]
    for name, n, wm, wmed, bm, tot in op_table(plan, trace):
        lines.append(f"{name:>10} {n:6d} {wm:10.2f} {wmed:9.2f} {bm:10.2f} {tot:12.1f}")
    L = int((plan.instrs[:, 0] >> 8).max())
    for layer in sorted({0, L // 2, max(L - 1, 0)}):
        lines.append(f"layer {layer}: op  first_ready  last_ready  last_done (us)")
        for name, a, b, c in layer_phases(plan, trace, layer):
            lines.append(f"   {name:>10} {a:10.1f} {b:10.1f} {c:10.1f}")
    return "\n".join(lines)
