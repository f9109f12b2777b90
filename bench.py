"""Benchmark of the fused MoE forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_8e] [--shapes workloads|table|none]

A step is one pass of the whole hot path over one batch: moe_route (softmax,
top-k, renormalisation) then moe_forward (grouping, GEMM1+SwiGLU, GEMM2 with
the weighted top-k sum, plus a fixed-order combine pass for top-k > 2 -- or
the small-T GEMV path) on synthetic inputs with the shapes and
distributions of the atrex-bench #009 "fused_moe" workload.  The headline
workload is "prefill, few large experts" (T=1979, H=2048, I=2048, E=8,
top-k 2); the other workloads are reported under "per_shape" (--shapes table:
every row of the atrex-bench #009 shapes table, plus a two-token decode).

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronise on both sides; each step is timed with CUDA events on the
launching stream, and a 256 MiB buffer is written between steps (untimed) so
that every step starts with a cold L2 (then 256 MiB are read, so
that L2 holds clean lines only: the step does not pay for writing back the
flush's dirty lines).  Multi-GPU (torchrun): one independent
replica per GPU, no collective in the data path; the time is the max over
ranks and `value` counts the work of all ranks.

--impl reference times the fp64 CPU oracle (formulation A, the per-token
loop) on the host cores, on a bounded sample of tokens of the same workload
per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import (SHAPES, TABLE_SHAPES, MoEShape, make_fp8_weights,  # noqa: E402
                        make_shape_inputs, PAGE_T_PROD_US as TABLE_T_PROD_US)

METRIC = "fused-MoE µs/call, TFLOP/s and % of roofline per shape; T=1 decode HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# T_Prod of the production op on the page's "XPU-A" hardware (atrex-bench #009 shapes table)
PAGE_T_PROD_US = {"prefill_8e": 772.50, "decode": 116.90, "prefill_thin": 5690.0,
                  "prefill_big": 18640.0}
FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def algorithmic_bytes(s: MoEShape, n_active: int, fp8_block: int = 0) -> float:
    """Activated expert weights (bf16, or FP8 codes plus one fp32 scale per
    block) + bf16 hidden + ids/weights + fp32 output."""
    n_w = n_active * 3.0 * s.H * s.I
    w_bytes = n_w * 2 if fp8_block == 0 else n_w + n_w / fp8_block * 4
    return w_bytes + s.T * s.H * 2 + s.T * s.k * 8 + s.T * s.H * 4


def roofline_us(s: MoEShape, n_active: int, peaks, fp8_block: int = 0) -> tuple[float, str]:
    t_flop = s.flops / (peaks["bf16_tflops"] * 1e12) * 1e6
    t_mem = algorithmic_bytes(s, n_active, fp8_block) / (peaks["hbm_gbs"] * 1e9) * 1e6
    return (t_flop, "tensor") if t_flop >= t_mem else (t_mem, "hbm")


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, device) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Throughput of all replicas: every rank did `steps` steps; the job took
    the slowest rank's time."""
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples (the JSON line carries their summary)
        out_dir = os.environ.get("MOE_BENCH_CLOCKS_DIR", tempfile.gettempdir())
        self.path = os.path.join(out_dir, f"moe_bench_clocks_gpu{gpu_index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
                except ValueError:
                    continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        max_mhz = max(r[1] for r in rows)
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3][1:5])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max_mhz,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded)}


# ------------------------------------------------------------------ our arm
def time_steps(step, K, W, flush, stream, marks=1):
    """Run W warm-up and K timed steps; step(ev_list) records events itself.
    Returns a list of per-step lists of elapsed ms between consecutive marks."""
    for _ in range(W):
        flush()
        step(None)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(marks + 1)] for _ in range(K)]
    for i in range(K):
        flush()
        step(evs[i])
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    return [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(marks)] for i in range(K)]


def traffic_from_profile(kernel: str, workload: str, launches_per_call: int = 1):
    """DRAM bytes per launch from the committed ncu summary, if its kernel
    source hash still matches the current source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    try:
        with open(path) as f:
            prof = json.load(f)
        h = hashlib.sha256()
        for src in prof["source_files"]:
            with open(os.path.join(ROOT, src), "rb") as sf:
                h.update(sf.read())
        if h.hexdigest() != prof["source_sha256"]:
            return None
        return float(prof["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def run_ours(args, ws, rank, local):
    import mixture_experts_expert_softmax_b200 as moe
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    s = SHAPES[args.workload]
    hidden, w1, w2, logits = make_shape_inputs(s, seed=0, device=str(dev))
    fp8 = args.weights == "fp8"
    if fp8:
        q1, s1, q2, s2 = make_fp8_weights(s.E, s.H, s.I, args.fp8_block, seed=0, device=str(dev))
        del w1, w2

        def forward(h, wts_, ids_, out_):
            moe.moe_forward_fp8(h, q1, s1, q2, s2, args.fp8_block, wts_, ids_, out_)
    else:
        def forward(h, wts_, ids_, out_):
            moe.moe_forward(h, w1, w2, wts_, ids_, out_)
    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_read = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    ids = torch.empty(s.T, s.k, dtype=torch.int32, device=dev)
    wts = torch.empty(s.T, s.k, dtype=torch.float32, device=dev)
    out = torch.empty(s.T, s.H, dtype=torch.float32, device=dev)

    def flush():
        # evict everything: write 256 MiB (twice L2), then read another
        # 256 MiB so that L2 holds only clean lines when the step starts
        flush_buf.zero_()
        flush_read.sum()

    def step(ev):
        if ev is not None:
            ev[0].record(stream)
        moe.moe_route(logits, s.k, True, ids, wts)
        if ev is not None:
            ev[1].record(stream)
        forward(hidden, wts, ids, out)
        if ev is not None:
            ev[2].record(stream)

    with ClockSampler(local) as clk:
        t = time_steps(step, args.steps, args.warmup, flush, stream, marks=2)
    route_ms = [x[0] for x in t]
    fwd_ms = [x[1] for x in t]
    total_ms = sum(a + b for a, b in t)
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(s.flops, args.steps, ws, total_ms)
    n_active = int(torch.unique(ids).numel())

    # per-kernel durations: the same K steps again with the library's event
    # profiler on (it records an event pair around every kernel launch)
    moe.profile_reset()
    moe.profile_enable(True)
    time_steps(step, args.steps, 1, flush, stream, marks=2)
    moe.profile_enable(False)
    prof = moe.profile_read()
    launches_per_step = sum(n for n, _ in prof.values()) / (args.steps + 1)
    kernels = {k: {"launches": n, "avg_us": ms * 1e3 / n} for k, (n, ms) in prof.items()}
    top = max(kernels, key=lambda k: kernels[k]["avg_us"] * kernels[k]["launches"])
    gemm1_flops = 4.0 * s.T * s.k * s.H * s.I
    gemm2_flops = 2.0 * s.T * s.k * s.H * s.I
    kernel_flops = {"gemm1_swiglu": gemm1_flops, "gemm2": gemm2_flops,
                    "gemm_fused": gemm1_flops + gemm2_flops}
    if top in kernel_flops:
        achieved = kernel_flops[top] / (kernels[top]["avg_us"] * 1e-6) / 1e12
        roof = {"kernel": top, "bound": "tensor", "achieved": round(achieved, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16_tflops"], 4),
                "peak_source": f"{peaks['source']} bf16 dense (burst)",
                "traffic": None if fp8 else traffic_from_profile(top, args.workload),
                "algorithmic_flops_per_launch": kernel_flops[top]}
    else:
        gb = algorithmic_bytes(s, n_active, args.fp8_block if fp8 else 0)
        achieved = gb / (kernels[top]["avg_us"] * 1e-6) / 1e9
        roof = {"kernel": top, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": f"{peaks['source']} HBM copy",
                "traffic": None if fp8 else traffic_from_profile(top, args.workload)}

    # end to end through the public API with host buffers
    h_hidden = hidden.cpu().pin_memory()
    h_logits = logits.cpu().pin_memory()
    h_out = torch.empty(s.T, s.H, dtype=torch.float32).pin_memory()
    d_hidden = torch.empty_like(hidden)
    d_logits = torch.empty_like(logits)

    def step_e2e(ev):
        if ev is not None:
            ev[0].record(stream)
        d_hidden.copy_(h_hidden, non_blocking=True)
        d_logits.copy_(h_logits, non_blocking=True)
        moe.moe_route(d_logits, s.k, True, ids, wts)
        forward(d_hidden, wts, ids, out)
        h_out.copy_(out, non_blocking=True)
        if ev is not None:
            ev[1].record(stream)

    te = time_steps(step_e2e, args.steps, args.warmup, flush, stream, marks=1)
    e2e_ms = max_over_ranks(sum(x[0] for x in te), dev)
    e2e_value = whole_job_tflops(s.flops, args.steps, ws, e2e_ms)
    h2d = h_hidden.numel() * 2 + h_logits.numel() * 4
    d2h = h_out.numel() * 4

    if args.timeline and rank == 0:
        # one more forward of the workload (cold L2) with the kernels'
        # per-tile / per-phase records on, written with their summary
        flush()
        torch.cuda.synchronize(dev)
        moe.timeline_start(1 << 16, device=dev)
        forward(hidden, wts, ids, out)
        recs = moe.timeline_stop()
        with open(args.timeline, "w") as f:
            json.dump({"workload": args.workload, "summary": moe.timeline_summary(recs),
                       "records": recs}, f)

    per_shape = {}
    fb = args.fp8_block if fp8 else 0
    if args.shapes == "workloads":
        per_shape = measure_shapes(moe, dev, peaks, flush, stream, SHAPES, PAGE_T_PROD_US,
                                   fp8_block=fb)
    elif args.shapes == "table":
        per_shape = measure_shapes(moe, dev, peaks, flush, stream, TABLE_SHAPES, TABLE_T_PROD_US,
                                   fp8_block=fb)

    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "us_per_call": round(statistics.median(fwd_ms) * 1e3, 2),
        "route_us": round(statistics.median(route_ms) * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8-e4m3 weights, bf16 activations" if fp8 else "bf16",
        "data": "synthetic (seeded randn, shapes and scales of atrex-bench #009 input.py)",
        "config": {"workload": s.name, "T": s.T, "H": s.H, "I": s.I, "E": s.E, "top_k": s.k,
                   "renorm": True, "active_experts": n_active,
                   "weights": (f"fp8 e4m3 codes, fp32 scale per {args.fp8_block} contraction "
                               "elements" if fp8 else "bf16"),
                   "l2": "flushed between steps (256 MiB write + 256 MiB read, untimed)",
                   "step": "moe_route + " + ("moe_forward_fp8" if fp8 else "moe_forward"),
                   "parallelism": f"replicas x{ws}"},
        "roofline": roof,
        "kernels": {k: {"launches": v["launches"], "avg_us": round(v["avg_us"], 2)}
                    for k, v in kernels.items()},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
        "peaks": {k: v for k, v in peaks.items()},
    }
    if args.workload in PAGE_T_PROD_US:
        page_tflops = s.flops / (PAGE_T_PROD_US[args.workload] * 1e-6) / 1e12
        line["vs_baseline"] = round(value / ws / page_tflops, 3)
        line["vs_baseline_ref"] = (f"T_Prod {PAGE_T_PROD_US[args.workload]} us on the page's "
                                   f"XPU-A (atrex-bench #009), = {page_tflops:.1f} TFLOP/s per GPU")
    if per_shape:
        line["per_shape"] = per_shape
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        wa, wb = ((q1, s1, args.fp8_block), (q2, s2, args.fp8_block)) if fp8 else (w1, w2)
        line["cpu_baseline"] = cpu_baseline(s, hidden, wa, wb, logits, budget_s=args.cpu_seconds)
    return line


def measure_shapes(moe, dev, peaks, flush, stream, shapes, page_us, K=10, W=3, fp8_block=0):
    """Forward-only time per shape; FP8 E4M3 weights when fp8_block > 0."""
    res = {}
    for name, s in shapes.items():
        if fp8_block and (s.H % fp8_block or s.I % fp8_block or fp8_block % 128):
            res[name] = {"skipped": f"block {fp8_block} does not divide H={s.H} and I={s.I}"}
            continue
        hidden, w1, w2, logits = make_shape_inputs(s, seed=0, device=str(dev))
        if fp8_block:
            q1, s1, q2, s2 = make_fp8_weights(s.E, s.H, s.I, fp8_block, seed=0, device=str(dev))
        ids, wts = moe.moe_route(logits, s.k, True)
        out = torch.empty(s.T, s.H, dtype=torch.float32, device=dev)

        def step(ev):
            if ev is not None:
                ev[0].record(stream)
            if fp8_block:
                moe.moe_forward_fp8(hidden, q1, s1, q2, s2, fp8_block, wts, ids, out)
            else:
                moe.moe_forward(hidden, w1, w2, wts, ids, out)
            if ev is not None:
                ev[1].record(stream)

        t = time_steps(step, K, W, flush, stream, marks=1)
        us = statistics.median(x[0] for x in t) * 1e3
        n_active = int(torch.unique(ids).numel())
        t_roof, bound = roofline_us(s, n_active, peaks, fp8_block)
        res[name] = {"T": s.T, "H": s.H, "I": s.I, "E": s.E, "k": s.k,
                     "us_per_call": round(us, 2),
                     "tflops": round(s.flops / (us * 1e-6) / 1e12, 2),
                     "hbm_gbs": round(algorithmic_bytes(s, n_active, fp8_block) / (us * 1e-6) / 1e9,
                                      1),
                     "roofline_bound": bound, "roofline_us": round(t_roof, 2),
                     "roofline_frac": round(t_roof / us, 4)}
        if name in page_us:
            res[name]["page_t_prod_us"] = page_us[name]
        del hidden, w1, w2, logits, ids, wts, out
        if fp8_block:
            del q1, s1, q2, s2
        torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ oracle (CPU)
def oracle_sample(s, hidden, w1, w2, logits, rows):
    """Seconds of the oracle's forward on the listed tokens; w1/w2 are the
    bf16 weights, or (codes, scales, block) triples of FP8 weights."""
    import oracle
    sel = torch.as_tensor(rows, dtype=torch.long)
    ids, w = oracle.route(logits[sel].numpy(), s.k, True)
    h = hidden[sel]
    t0 = time.perf_counter()
    if isinstance(w1, tuple):
        (q1, s1, block), (q2, s2, _) = w1, w2
        oracle.moe_token_loop_fp8(h, q1, s1, q2, s2, block, w, ids)
    else:
        oracle.moe_token_loop(h, w1, w2, w, ids)
    return time.perf_counter() - t0


def calibrate_rows(s, hidden, w1, w2, logits, budget_s):
    """Number of tokens whose oracle forward takes about budget_s."""
    import oracle
    threads = oracle.max_threads()
    n0 = min(s.T, max(1, threads))
    dt = oracle_sample(s, hidden, w1, w2, logits, np.arange(n0))
    n = int(max(1, min(s.T, n0 * budget_s / max(dt, 1e-6))))
    return n, threads


def cpu_baseline(s, hidden, w1, w2, logits, budget_s=10.0):
    import oracle

    def host(w):
        return tuple(x.cpu() if torch.is_tensor(x) else x for x in w) if isinstance(w, tuple) \
            else w.cpu()

    hidden, w1, w2, logits = hidden.cpu(), host(w1), host(w2), logits.cpu()
    n, threads = calibrate_rows(s, hidden, w1, w2, logits, budget_s)
    rows = np.arange(n)
    dt = oracle_sample(s, hidden, w1, w2, logits, rows)
    flops = 6.0 * n * s.k * s.H * s.I
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"oracle formulation A (fp64 per-token loop) on the first {n} of {s.T} "
                      f"tokens of the same workload ({dt:.1f} s, {threads} OpenMP threads)",
            "cpu": _cpu_name()}


def _cpu_name():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, ws, rank):
    if rank != 0:
        return None
    import oracle
    s = SHAPES[args.workload]
    hidden, w1, w2, logits = make_shape_inputs(s, seed=0, device="cpu")
    if args.weights == "fp8":
        # the oracle's FP8 formulation on the same codes and scales
        q1, s1, q2, s2 = make_fp8_weights(s.E, s.H, s.I, args.fp8_block, seed=0, device="cpu")
        w1, w2 = (q1, s1, args.fp8_block), (q2, s2, args.fp8_block)
    per_step = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    n, threads = calibrate_rows(s, hidden, w1, w2, logits, per_step)
    rows = np.arange(n)
    for _ in range(args.warmup):
        oracle_sample(s, hidden, w1, w2, logits, rows)
    total = 0.0
    for _ in range(args.steps):
        total += oracle_sample(s, hidden, w1, w2, logits, rows)
    flops = 6.0 * n * s.k * s.H * s.I * args.steps
    value = flops / total / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded randn, shapes and scales of atrex-bench #009 input.py)",
        "config": {"workload": s.name, "T": s.T, "H": s.H, "I": s.I, "E": s.E, "top_k": s.k,
                   "renorm": True, "weights": args.weights,
                   "step": f"oracle forward of a {n}-token sample"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"{n} of {s.T} tokens per step, fp64 per-token loop",
                         "cpu": _cpu_name()},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(SHAPES), default="prefill_8e")
    ap.add_argument("--shapes", choices=["workloads", "table", "none"], default="workloads",
                    help="per-shape table: the five workloads, every row of the page's "
                         "shapes table, or none")
    ap.add_argument("--no-shapes", action="store_true", help="same as --shapes none")
    ap.add_argument("--weights", choices=["bf16", "fp8"], default="bf16",
                    help="expert weights: bf16, or FP8 E4M3 codes with fp32 scales per "
                         "--fp8-block contraction elements (moe_forward_fp8)")
    ap.add_argument("--fp8-block", type=int, default=128)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--timeline", metavar="PATH",
                    help="after the timed steps, write the kernels' per-tile / per-phase "
                         "records of one more forward (moe_timeline) to PATH as JSON")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.no_shapes:
        args.shapes = "none"
    ws, rank, local = dist_env()
    if args.impl == "reference":
        line = run_reference(args, ws, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        line = run_ours(args, ws, rank, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
