"""Decode-step benchmark of the persistent megakernel on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config dense-8b] [--impl mk|reference]

A step is one decode step of the whole model (every layer, LM head) for the
batch, through the C ABI (mk_decode_step).  Inputs are seeded and synthetic
(random-init weights of the named shape, prefilled KV cache, uniform token ids,
teacher forcing).  One JSON line on stdout (rank 0):

  value   decode tokens/s with inputs resident in HBM (CUDA events on the launching stream,
          K consecutive steps, max over ranks)
  e2e     the same metric with tokens/positions/lengths copied from pinned host memory and
          the logits copied back inside the timed region
  roofline / mbu
          algorithmic bytes per step (bf16 weights read + KV-cache positions read/written)
          / kernel time, against the measured HBM copy bandwidth (MEASURED_PEAKS.json) and
          against the 8 TB/s B200 specification
  cpu_baseline
          the CPU oracle (single-threaded fp64) on a bounded sample of the same step

Multi-GPU (torchrun): independent replicas, one model per GPU, no collective on the data
path; value = tokens/s summed over ranks, timed as the slowest rank.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import fixtures as fx  # noqa: E402

METRIC = "decode tokens/s (batch tokens per decode step / step time)"
SPEC_HBM_GBS = 8000.0
# the default line's workload, then the other configurations it reports under "per_config"
MAIN_CONFIG = "dense-8b"
PER_CONFIG = ("dense-0.6b", "dense-13b-b8", "moe-128x8")
FALLBACK_HBM_GBS = 6650.0


def weight_bytes_read(cfg) -> int:
    """bf16 weight bytes a step reads apart from MoE experts: every layer matrix and norm (MoE: the
    router instead of the MLP), the LM head, B embedding rows."""
    H, L = cfg.hidden, cfg.n_layers
    per = 2 * H + cfg.q_dim * H * 2 + cfg.kv_dim * H * 2
    per += cfg.n_experts * H if cfg.n_experts else 3 * cfg.ffn_dim * H
    if cfg.qk_norm:
        per += 2 * cfg.head_dim
    return 2 * (L * per + H + cfg.vocab * H + cfg.batch * H)


def expert_bytes_read(cfg, distinct_per_step) -> float:
    """MoE: bf16 bytes of the distinct picked experts' gate, up and down matrices (each read once)."""
    return 2.0 * 3 * cfg.expert_ffn_dim * cfg.hidden * float(np.mean(distinct_per_step))


def kv_bytes(cfg, seq_lens) -> int:
    """KV-cache bytes a step touches: S_b cached positions read + 1 new row written, K and V, all layers."""
    return 2 * cfg.n_layers * cfg.n_kv_heads * cfg.head_dim * 2 * int(np.sum(np.asarray(seq_lens) + 1))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "auto_regressive_decode_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch of the full workload, scaled from a committed ncu capture of its small case
    (`--layers`) by the algorithmic bytes, if that capture was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_source") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this process's GPU, sampled during the timed region.

    NVML is polled from a thread every 5 ms (read-only queries); without NVML, nvidia-smi -lms."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.samples = []  # (sm_mhz, max_mhz, {reason names})
        self.proc = None
        self.stop = threading.Event()
        self.t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def poll():
                while not self.stop.is_set():
                    r = get_reasons(h)
                    self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx,
                                         {k for k, bit in self.REASONS.items() if r & bit}))
                    self.stop.wait(0.005)

            self.t = threading.Thread(target=poll, daemon=True)
            self.t.start()
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7 or not f[0].replace(".", "").isdigit():
                continue
            self.samples.append((float(f[0]), float(f[1]) if f[1].replace(".", "").isdigit() else None,
                                 {names[i] for i in range(4) if f[3 + i].lower() == "active"}))

    def __exit__(self, *a):
        self.stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t:
            self.t.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[0]) for s in self.samples]
        mx = [float(s[1]) for s in self.samples if s[1]]
        reasons = sorted(set().union(*(s[2] for s in self.samples)))
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample of the step
# ---------------------------------------------------------------------------------------------------------

def cpu_baseline(cfg, seed=fx.DEFAULT_SEED, max_layers=2):
    import oracle as ora
    from tests.helpers import expert_loader, host_model
    n = min(max_layers, cfg.n_layers)
    g, ls = host_model(cfg, seed, layers=range(n))
    S = fx.context_lengths(cfg, seed)
    kc = [fx.kv_prefill(cfg, l, 0, S, seed) for l in range(n)]
    vc = [fx.kv_prefill(cfg, l, 1, S, seed) for l in range(n)]
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls,
                      expert_loader(cfg, seed) if cfg.n_experts else None)
    tok = fx.tokens(cfg, seed)[0]
    x = fx.bf16_to_f32(g["embed"][tok]).astype(np.float64)
    t0 = time.perf_counter()
    for l in range(n):
        model.layer_forward(l, x, kc[l], vc[l], S, S)
    t_layers = (time.perf_counter() - t0) / n
    t1 = time.perf_counter()
    for b in range(cfg.batch):
        model.lm_head(x[b])
    t_head = time.perf_counter() - t1
    step_s = t_layers * cfg.n_layers + t_head
    return {"value": cfg.batch / step_s, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} of {cfg.n_layers} layers + LM head of step 0 (fp64, single thread), "
                      f"extrapolated to the full step: {step_s:.3f} s/step",
            "step_s": step_s}


def max_over_ranks(values, world, device="cpu"):
    """Each value's maximum over the ranks (a job's time is its slowest rank's); identity for one rank."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_tokens_per_s(world, batch, steps, total_ms):
    """Whole-job tokens/s: every rank (replica) decodes `batch` tokens per step."""
    return world * batch * steps / (total_ms / 1e3)


def run_reference(args, cfg, rank):
    """The oracle timed on the host.  Each timed step is a bounded sample: one of the L layers of the
    decode step (layers taken in turn).  `ms_per_step` and `steps` report those samples as timed; the
    throughput extrapolates the median layer to the whole step (L layers plus the LM head, timed once)."""
    if rank != 0:
        return
    import oracle as ora
    from tests.helpers import expert_loader, host_model
    n_lay = min(2, cfg.n_layers)
    g, ls = host_model(cfg, layers=range(n_lay))
    S = fx.context_lengths(cfg)
    kc = [fx.kv_prefill(cfg, l, 0, S) for l in range(n_lay)]
    vc = [fx.kv_prefill(cfg, l, 1, S) for l in range(n_lay)]
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls,
                      expert_loader(cfg) if cfg.n_experts else None)
    tok = fx.tokens(cfg)[0]
    x = fx.bf16_to_f32(g["embed"][tok]).astype(np.float64)
    times = []
    for i in range(args.warmup + args.steps):
        l = i % n_lay
        t0 = time.perf_counter()
        model.layer_forward(l, x.copy(), kc[l], vc[l], S, S)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    t0 = time.perf_counter()
    for b in range(cfg.batch):
        model.lm_head(x[b])
    t_head = time.perf_counter() - t0
    layer_s = statistics.median(times)
    step_s = layer_s * cfg.n_layers + t_head
    value = cfg.batch / step_s
    out = {"impl": "reference", "metric": METRIC,
           "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": layer_s * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(cfg),
           "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "1 GPU",
           "timed_unit": f"one of the {cfg.n_layers} layers of the decode step per timed step (a bounded "
                         f"sample); value extrapolates: median layer x {cfg.n_layers} + LM head "
                         f"= {step_s * 1e3:.1f} ms per decode step",
           "extrapolated_ms_per_decode_step": step_s * 1e3,
           "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": "tokens/s",
                            "sample": f"each timed step: one of {cfg.n_layers} layers (fp64, single thread); "
                                      f"decode step = median layer x {cfg.n_layers} + LM head = {step_s:.3f} s"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def workload_config(cfg, paged=False):
    """The workload a line measures; the same dict in both arms."""
    ctx = f"ctx U[{cfg.ctx_lo},{cfg.ctx_hi}]" if cfg.ragged else f"ctx {cfg.ctx}"
    out = {"workload": f"{cfg.name}: {cfg.n_layers} layers, hidden {cfg.hidden}, {cfg.n_q_heads}q/{cfg.n_kv_heads}kv "
                       f"heads x {cfg.head_dim}, ffn {cfg.ffn_dim or cfg.expert_ffn_dim}, vocab {cfg.vocab}; "
                       f"batch {cfg.batch}, {ctx}, teacher-forced decode",
           "batch": cfg.batch, "max_ctx": cfg.max_ctx, "weights": "bf16 ~N(0,0.02), seeded",
           "kv_cache": "bf16 ~N(0,1), seeded", "accumulate": "fp32",
           "l2": "inputs larger than L2 (weights stream from HBM every step)"}
    if paged:
        out["kv_layout"] = f"paged, {32768 // (2 * cfg.head_dim)}-position pages in a shuffled pool"
    return out


# ---------------------------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------------------------

def make_decoder(cfg, seed, dev, paged):
    """Seeded device weights and caches of cfg and a Decoder on them (the cache as a shuffled page pool
    when paged)."""
    import torch
    import auto_regressive_decode_b200.mk as mk
    from fixtures.device import device_caches, device_model
    S0 = fx.context_lengths(cfg, seed)
    w = device_model(cfg, seed)
    kc, vc = device_caches(cfg, S0, seed)
    if not paged:
        return mk.Decoder(cfg, w, kc, vc), S0
    # one attention stage per page, pages in a seeded random order
    page = 32768 // (2 * cfg.head_dim)
    stride = -(-cfg.max_ctx // page)
    table = np.random.default_rng(seed).permutation(cfg.batch * stride).reshape(cfg.batch, stride)
    pools = []
    for c in (kc, vc):
        L, B_, nkv, T, hd = c.shape
        pool = torch.empty((L, cfg.batch * stride, nkv, page, hd), dtype=c.dtype, device=c.device)
        for b in range(B_):
            for j in range(stride):
                lo, hi = j * page, min(T, (j + 1) * page)
                pool[:, int(table[b, j]), :, :hi - lo] = c[:, b, :, lo:hi]
        pools.append(pool)
    del kc, vc
    d_table = torch.from_numpy(table.astype(np.int32)).to(dev)
    return mk.Decoder(cfg, w, pools[0], pools[1], block_table=d_table, page_size=page), S0


def measure(args, cfg, rank, world, dev, full=True):
    """Time args.steps decode steps of cfg after args.warmup untimed ones (CUDA events on the launching
    stream, max over ranks).  full: also the end-to-end (host buffers) and greedy-loop numbers."""
    import torch
    import auto_regressive_decode_b200.mk as mk

    seed = fx.DEFAULT_SEED + rank
    dec, S0 = make_decoder(cfg, seed, dev, args.paged)
    toks = fx.tokens(cfg, seed)
    B, V = cfg.batch, cfg.vocab
    n_total = args.warmup + args.steps
    # per-step inputs, resident on the device (teacher forcing; positions wrap after cfg.steps)
    steps_idx = np.arange(n_total) % cfg.steps
    all_tok = torch.from_numpy(toks[steps_idx].astype(np.int32)).to(dev)
    all_len = torch.from_numpy((S0[None, :] + steps_idx[:, None]).astype(np.int32)).to(dev)
    logits = torch.empty((B, V), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def check():
        st = dec.status()
        if st != 0:
            raise RuntimeError(f"{cfg.name}: device status {mk.mk_status_string(st)}")

    for i in range(args.warmup):
        dec.step(all_tok[i], all_len[i], all_len[i], logits)
    torch.cuda.synchronize()
    check()

    # ---- device-resident timing: one event pair per step, on the launching stream
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    props = torch.cuda.get_device_properties(dev)
    uuid = "GPU-" + str(props.uuid) if not str(props.uuid).startswith("GPU-") else str(props.uuid)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(uuid) as clk:
        ev[0].record(stream)
        for j in range(args.steps):
            i = args.warmup + j
            dec.step(all_tok[i], all_len[i], all_len[i], logits)
            ev[j + 1].record(stream)
        torch.cuda.synchronize()
    barrier()
    check()
    per_step_ms = [ev[j].elapsed_time(ev[j + 1]) for j in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])

    # ---- MoE: the distinct experts each timed step read (its routing, replayed untimed)
    distinct = []
    if cfg.n_experts:
        for j in range(args.steps):
            i = args.warmup + j
            dec.step(all_tok[i], all_len[i], all_len[i], logits)
            distinct.append(int(dec.routing()[3].sum()))

    e2e_ms = greedy_ms = float("nan")
    if full:
        # ---- end to end through the C ABI with host buffers
        h_tok = torch.from_numpy(toks[steps_idx].astype(np.int32)).pin_memory()
        h_len = torch.from_numpy((S0[None, :] + steps_idx[:, None]).astype(np.int32)).pin_memory()
        h_logits = torch.empty((B, V), dtype=torch.float32).pin_memory()
        d_tok = torch.empty(B, dtype=torch.int32, device=dev)
        d_len = torch.empty(B, dtype=torch.int32, device=dev)
        d_pos = torch.empty(B, dtype=torch.int32, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for j in range(args.steps):
            i = args.warmup + j
            d_tok.copy_(h_tok[i], non_blocking=True)
            d_len.copy_(h_len[i], non_blocking=True)
            d_pos.copy_(h_len[i], non_blocking=True)
            dec.step(d_tok, d_pos, d_len, logits)
            h_logits.copy_(logits, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = e0.elapsed_time(e1)
        check()

        # ---- on-device greedy decoding: K steps in one call, each step's arg-max fed back on the device
        # (after the MoE replay: the loop rewrites cache rows below S0 to make room)
        picks = torch.empty((args.steps, B), dtype=torch.int32, device=dev)
        g_len = torch.from_numpy(np.maximum(S0 - args.steps, 0).astype(np.int32)).to(dev)  # room for K steps
        g_tok = all_tok[0].clone()
        dec.greedy(3, g_tok, g_len, picks)  # warm-up
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        dec.greedy(args.steps, g_tok, g_len, picks)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        greedy_ms = e0.elapsed_time(e1)
        check()

    # ---- max over ranks
    total_ms, e2e_ms, greedy_ms = max_over_ranks([total_ms, e2e_ms, greedy_ms], world, dev)
    dec.close()
    del dec, all_tok, all_len, logits
    torch.cuda.empty_cache()

    ms = total_ms / args.steps
    lens = [S0 + (k % cfg.steps) for k in range(args.warmup, n_total)]
    bytes_step = weight_bytes_read(cfg) + float(np.mean([kv_bytes(cfg, s) for s in lens]))
    if cfg.n_experts:
        bytes_step += expert_bytes_read(cfg, distinct)
    peak, peak_kind = measured_peaks()
    achieved = bytes_step / (ms / 1e3) / 1e9
    r = {
        "workload": workload_config(cfg)["workload"],
        "ms_per_step": ms,
        "tokens_per_s": job_tokens_per_s(world, B, args.steps, total_ms),
        "step_latency_ms": {"median": statistics.median(per_step_ms), "p10": float(np.percentile(per_step_ms, 10)),
                            "p90": float(np.percentile(per_step_ms, 90))},
        "bytes_per_step": bytes_step,
        **({"moe_distinct_experts_per_layer": float(np.mean(distinct)) / cfg.n_layers} if cfg.n_experts else {}),
        "mbu": {"vs_spec_8tbs": achieved / SPEC_HBM_GBS, f"vs_{peak_kind}_{peak:.0f}gbs": achieved / peak},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback", "traffic": ncu_traffic(cfg.name), "kernel": "mk_persistent"},
        "clocks": clk.summary(),
    }
    if full:
        r["e2e_ms"] = e2e_ms
        r["greedy_ms"] = greedy_ms
    return r


def run_mk(args, cfg, rank, world):
    import torch

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    m = measure(args, cfg, rank, world, dev, full=True)
    per_config = {}
    if args.per_config and not args.layers and cfg.name == MAIN_CONFIG:
        for name in PER_CONFIG:
            c = fx.CONFIGS[name]
            pc = measure(args, c, rank, world, dev, full=False)
            per_config[name] = {k: pc[k] for k in ("workload", "ms_per_step", "tokens_per_s", "step_latency_ms",
                                                   "bytes_per_step", "mbu", "roofline", "clocks")}
            if c.n_experts:
                per_config[name]["moe_distinct_experts_per_layer"] = pc["moe_distinct_experts_per_layer"]
    if rank != 0:
        return
    B, V = cfg.batch, cfg.vocab
    out = {
        "metric": METRIC,
        "value": m["tokens_per_s"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights and KV cache, uniform token ids)",
        "config": workload_config(cfg, args.paged),
        "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
        "step_latency_ms": m["step_latency_ms"],
        "bytes_per_step": m["bytes_per_step"],
        **({"moe_distinct_experts_per_layer": m["moe_distinct_experts_per_layer"]} if cfg.n_experts else {}),
        "mbu": m["mbu"],
        "roofline": m["roofline"],
        "e2e": {"value": job_tokens_per_s(world, B, args.steps, m["e2e_ms"]), "unit": "tokens/s",
                "h2d_bytes_per_step": 3 * 4 * B, "d2h_bytes_per_step": 4 * B * V},
        "greedy_loop": {"value": job_tokens_per_s(world, B, args.steps, m["greedy_ms"]), "unit": "tokens/s",
                        "note": "mk_decode_greedy: K steps in one call, arg-max fed back on the device"},
        "gpu_launches": args.steps,
        "clocks": m["clocks"],
    }
    if per_config:
        out["per_config"] = per_config
    if not args.no_cpu_baseline and world == 1:  # the oracle baseline: rank 0 at one GPU only
        base = cpu_baseline(cfg)
        out["cpu_baseline"] = {k: base[k] for k in ("value", "unit", "cores", "kind", "sample")}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=MAIN_CONFIG, choices=sorted(fx.CONFIGS))
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the other configurations the default line reports under per_config")
    ap.add_argument("--paged", action="store_true", help="run the KV cache as a paged pool (block table)")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: the config with this many layers (same shapes); not a bench line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = fx.CONFIGS[args.config]
    if args.layers:
        cfg = cfg.replace(name=f"{cfg.name}-{args.layers}l", n_layers=args.layers)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_mk(args, cfg, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
