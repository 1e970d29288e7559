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


def layer_breakdown(plan, trace, layer):
    """Where one layer's time goes, per op: medians over the op's instructions of
    ready, prologue (ready -> inputs loaded), first stage (-> first weight stage
    landed), stream (-> last stage consumed), epilogue (-> done), done, the
    producer's first and last copy, and the op's last done.  Times in us, from
    the last done stamp of the layer before (layer 0: the step's first stamp);
    prologue .. epilogue are durations, the rest are points in time."""
    t = trace.astype(np.int64)
    ops = plan.instrs[:, 0] & 0xFF
    layers = plan.instrs[:, 0] >> 8
    prev = t[layers == layer - 1, 2].max() if layer > 0 and (layers == layer - 1).any() else t[:, 0].min()
    out = []
    for op in sorted(set(ops[layers == layer].tolist())):
        x = t[(ops == op) & (layers == layer)]
        med = lambda a: float(np.median(a)) / 1e3  # noqa: E731
        out.append({"op": OP_NAMES.get(op, str(op)), "n": int(len(x)), "ready": med(x[:, 1] - prev),
                    "prologue": med(x[:, 4] - x[:, 1]), "first_stage": med(x[:, 5] - x[:, 4]),
                    "stream": med(x[:, 6] - x[:, 5]), "epilogue": med(x[:, 2] - x[:, 6]), "done": med(x[:, 2] - prev),
                    "producer_first": med(x[:, 3] - prev), "producer_last": med(x[:, 7] - prev),
                    "done_max": float(x[:, 2].max() - prev) / 1e3})
    return out


def handoff_costs(plan, trace):
    """Per op: median time (us) from a signalling instruction's done stamp (the
    last of its op on an SM) to the start of the next instruction on the same
    SM -- its signal (barrier and release) and the fetch of the next instruction."""
    t = trace.astype(np.int64)
    ops = plan.instrs[:, 0] & 0xFF
    sig = plan.instrs[:, 3] >= 0
    off = np.asarray(plan.offsets)
    same = np.zeros(len(t), dtype=bool)
    for s in range(len(off) - 1):
        same[off[s]:off[s + 1] - 1] = True
    same &= sig
    gap = np.full(len(t), np.nan)
    gap[:-1] = (t[1:, 0] - t[:-1, 2]) / 1e3
    return {OP_NAMES.get(op, str(op)): float(np.median(gap[same & (ops == op)]))
            for op in sorted(set(ops.tolist())) if (same & (ops == op)).any()}


def format_breakdown(rows) -> str:
    keys = ("ready", "prologue", "first_stage", "stream", "epilogue", "done", "producer_first", "producer_last",
            "done_max")
    lines = [f"{'op':>10} {'n':>4} " + " ".join(f"{k:>14}" for k in keys)]
    for r in rows:
        lines.append(f"{r['op']:>10} {r['n']:4d} " + " ".join(f"{r[k]:14.2f}" for k in keys))
    return "\n".join(lines)


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


def main(argv=None):
    """Trace a few decode steps of a seeded workload on the GPU and print the timeline of some layers:
    python -m auto_regressive_decode_b200.trace --config dense-8b --layers 5 20"""
    import argparse
    import os
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="dense-8b")
    ap.add_argument("--layers", type=int, nargs="*", default=None)
    ap.add_argument("--steps", type=int, default=6)
    args = ap.parse_args(argv)
    os.environ["MK_TRACE"] = "1"  # read by mk_create
    import torch

    import fixtures as fx
    from fixtures.device import device_caches, device_model

    from . import mk
    cfg = fx.CONFIGS[args.config]
    S0, toks = fx.context_lengths(cfg), fx.tokens(cfg)
    dec = mk.Decoder(cfg, device_model(cfg), *device_caches(cfg, S0))
    plan = mk.Plan(mk.model_desc(cfg), torch.cuda.get_device_properties(0).multi_processor_count)
    logits = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    for k in range(args.steps):
        lens = torch.from_numpy((S0 + k).astype(np.int32)).cuda()
        dec.step(torch.from_numpy(toks[k % toks.shape[0]].copy()).cuda(), lens, lens, logits)
    torch.cuda.synchronize()
    if dec.status() != 0:
        raise RuntimeError("device status %d" % dec.status())
    t = mk.decoder_trace(dec)
    print(summarize(plan, t))
    print("hand-off (done -> next instruction start, us):", {k: round(v, 2) for k, v in handoff_costs(plan, t).items()})
    for layer in (args.layers if args.layers is not None else [cfg.n_layers // 2]):
        print(f"layer {layer} (us from the previous layer's last done; medians over instructions)")
        print(format_breakdown(layer_breakdown(plan, t, layer)))
    dec.close()


if __name__ == "__main__":
    main()
