#!/usr/bin/env python
"""Benchmark of libfattn on B200: one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --sweep          # section 9.2 matrix, one JSON line per point

A step is one pass of the prefill hot path (closed-form KV tile ranges, TMA
Q/K/V tiles, tcgen05 S = Q K^T, masked exp2 online softmax, P V, O / l and
LSE) over the causal 4 x 16 x 4096, d = 128 bf16 workload; ``value`` is its
in-mask TFLOP/s (4 d FLOPs per allowed (q, k) pair per head) with inputs
resident in HBM, the median of five timed regions of K steps (``repeats``).
The same run reports: that step with L2 flushed before every launch
(``cold_l2``); end to end on pinned host buffers (``e2e``); the backward with
recomputation (``bwd``) and the FP8 forward (``fp8``) on that workload; the
split-KV decode and its paged variant on the 64 x 32 x 32768 cache
(``decode``, ``decode_paged``, GB/s); the d = 64 causal, sliding-window,
long-causal and packed variable-length prefills (``extra``), each with its
roofline; the fp64 oracle on the host cores (``cpu_baseline``: all cores,
one core, sampled long workloads and decode slices with extrapolated full-run
times).  ``summary``, the last key, repeats the headline figures compactly.

Multi-GPU (torchrun, one rank per GPU): (batch, head) units are independent,
so every rank runs its own full copy of the workload with no collective on the
data path (weak scaling); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "attention fwd TFLOP/s (in-mask FLOPs) & % bf16 tensor peak; decode HBM GB/s"
HEADLINE = "causal_4k"
HEADLINE_D64 = "causal_4k_d64"
WINDOW_D64 = "window_bidir_32k_d64"
HEADLINE_REPEATS = 5
DECODE = "decode_32k"
EXTRA = ["window_bidir_32k", "window_causal_32k", "causal_64k_qscale"]
VARLEN_SEQS, VARLEN_MIN, VARLEN_MAX, VARLEN_H = 32, 256, 4096, 16  # packed batch of causal requests
PAGE_SIZE = 256  # paged-KV decode: tokens per page
PREFILL_KERNEL = "attn_fwd_sm100_kernel"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "attn_fwd_sm100_kernel": ["attn_fwd_sm100.cuh", "sched.cuh", "dev_prims.cuh"],
    "decode_split_kernel": ["decode_splitkv.cuh", "dev_prims.cuh"],
    "attn_bwd_sm100_kernel": ["attn_bwd_sm100.cuh", "sched.cuh", "dev_prims.cuh"],
    "attn_fwd_fp8": ["attn_fwd_sm100.cuh", "sched.cuh", "dev_prims.cuh"],
}


def _code_only(text: str) -> str:
    """C++ source without its comments and trailing blanks: an edit of a
    comment does not change what the kernel does."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_digest(kernel: str) -> str:
    """Digest of the code (comments removed) of the source files a kernel is
    compiled from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "io_aware_exact_34_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(kernel, {}).get(workload)
    if not ent or ent.get("source_digest") != kernel_source_digest(kernel):
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed regions."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, busy_power_w=300.0):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        busy = [r for r in rows if r[2] >= busy_power_w] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i, flag in enumerate(r[3]) if flag.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in busy), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(busy), "power_w_max": max(r[2] for r in rows), "reasons": reasons}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float) -> float:
    """The slowest rank's time: every rank gets the max (an all-reduce on the
    process group's device, CPU tensors for gloo)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base_seed: int, rank: int) -> int:
    """Each replica draws its own inputs of the same shape (weak scaling)."""
    return base_seed + rank


def timed(world, fn, steps, warmup):
    """Average device ms per step of fn over `steps`, CUDA events on the
    current stream, barrier + synchronize on both sides, max over ranks."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        fn()
    end.record()
    end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(world, start.elapsed_time(end) / steps)


REGIONS = 3          # burst regions per secondary line (--regions)
SUSTAINED = True     # time the sustained regime too (--no-sustained turns it off)


def timed_median(world, fn, steps, warmup, reps=None, gap_s=0.05, record=None):
    """Median over `reps` timed regions of `steps` steps each.  Before each
    region the device idles for `gap_s` of wall time and fn runs `warmup`
    (then 3) untimed times.  Back-to-back regions of a long kernel drift down
    to the power-capped clock within some tens of milliseconds; the idle gap
    keeps every region a burst measurement, the regime of the measured burst
    peak it is divided by, and the median keeps a region that caught a clock
    transition out of the line.  `timed_sustained` gives the other regime."""
    import torch
    reps = REGIONS if reps is None else reps
    out = []
    for r in range(reps):
        torch.cuda.synchronize()
        time.sleep(gap_s)
        out.append(timed(world, fn, steps, warmup if r == 0 else 3))
    if record is not None:
        record.extend(out)
    return statistics.median(out)


SOAK_S = 0.5


def timed_sustained(world, fn, steps, soak_s=SOAK_S):
    """One region of `steps` steps timed right after fn has run back to back,
    untimed, for `soak_s` of wall time: the clock the part settles at under its
    power cap.  It is divided by the measured sustained peak.  None when the
    sustained regime is switched off."""
    import torch
    if not SUSTAINED:
        return None
    t_end = time.perf_counter() + soak_s
    while time.perf_counter() < t_end:
        for _ in range(10):
            fn()
        torch.cuda.synchronize()
    return timed(world, fn, steps, 0)


def sustained_entry(world, ms, flops, peaks, scale=1.0):
    """The sustained figure of a TFLOP/s line against the measured sustained
    bf16 peak (times `scale` for another dtype)."""
    if ms is None:
        return None
    tf = flops / (ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"] * scale
    return {"value": world * tf, "unit": "TFLOP/s", "ms_per_step": ms, "soak_s": SOAK_S,
            "peak": peak, "frac": tf / peak, "peak_source": "bf16 dense, sustained" + (" x 2" if scale != 1.0 else "")}


def timed_cold_l2(world, fn, steps, warmup, flush):
    """Average device ms per step of fn when every step starts with a cold L2:
    a write of `flush` (larger than L2) precedes each step outside the events
    that bracket it.  Max over ranks."""
    import torch
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    barrier(world)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush.zero_()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(world, sum(a.elapsed_time(b) for a, b in evs) / steps)


def prefill_flops(fl, w):
    c = fl.attn_count_blocks(w.Lq, w.Lk, w.causal, w.window_left, w.window_right, 128, 128)
    return 4.0 * w.d * c["pairs"] * w.B * w.H, c


def tensor_roofline(achieved, peaks, peak_src, kernel, traffic, scale=1.0, scale_note=""):
    peak = peaks["bf16_tflops"] * scale
    src = f"{peak_src} bf16 dense (burst)" + scale_note
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": traffic, "peak_source": src, "kernel": kernel}


def exp_roofline(achieved, peaks, peak_src, d):
    """The exponential unit's ceiling on the same in-mask FLOPs: every allowed
    pair needs one exp2, which runs on the special-function unit at 16 per
    clock per SM, while the tensor core does 8192 dense bf16 FLOPs per clock
    per SM.  At 4*d FLOPs per pair the exp rate caps the kernel at
    16 * 4d / 8192 = d / 128 of the bf16 peak at the same clock, whatever the
    MMA precision: half of it at d = 64, and the bf16 peak itself for the FP8
    path at d = 128."""
    peak = peaks["bf16_tflops"] * d / 128.0
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"{peak_src} bf16 dense (burst) x d/128 (16 exp2/clk/SM vs 8192 bf16 FLOP/clk/SM)",
            "unit_bound": "MUFU ex2"}


def r4(x):
    """Four significant digits for the summary."""
    if x is None:
        return None
    return float(f"{x:.4g}")


# ---------------------------------------------------------------------- CPU baseline (the oracle)

def allowed_keys(w, rows_i):
    """Allowed keys of query rows rows_i (numpy int array) under w's mask:
    accounting of the work a sampled row costs, not attention arithmetic."""
    import numpy as np
    i = np.asarray(rows_i, dtype=np.int64)
    shift = w.Lk - w.Lq
    lo = np.zeros_like(i)
    hi = np.full_like(i, w.Lk - 1)
    if w.window_left >= 0:
        lo = np.maximum(lo, i + shift - w.window_left)
    wr = w.window_right
    if w.causal:
        wr = 0 if wr < 0 else min(wr, 0)
    if wr >= 0:
        hi = np.minimum(hi, i + shift + wr)
    return np.maximum(hi - lo + 1, 0)


def cpu_sampled(w, full_heads, n_random, seed=7):
    """The oracle on a stratified row sample of a long workload: every row of
    `full_heads`, plus first / last rows, tile and window edges and `n_random`
    random rows of every head.  Returns measured pairs/s and the full-run time
    extrapolated from it."""
    from io_aware_exact_34_b200 import synth
    from oracle import oracle
    q, k, v = synth.make_inputs(w)
    rows = synth.sample_rows(w, n_random=n_random, seed=seed, full_heads=full_heads).numpy()
    pairs = float(allowed_keys(w, rows[:, 2]).sum())
    t0 = time.perf_counter()
    oracle.attn_rows(q, k, v, rows, w.scale, w.causal, w.window_left, w.window_right)
    dt = time.perf_counter() - t0
    c = oracle.count_blocks(w.Lq, w.Lk, w.causal, w.window_left, w.window_right, 128, 128)
    total_pairs = float(c["pairs"]) * w.B * w.H
    pps = pairs / dt
    return {"pairs_per_s": pps, "tflops": 4.0 * w.d * pps / 1e12, "rows": int(rows.shape[0]),
            "full_heads": len(full_heads), "random_rows_per_head": n_random, "seconds": dt,
            "extrapolated_full_run_s": total_pairs / pps, "extrapolated": True}


def cpu_decode_slices(wd, n_slices, dev=None):
    """The oracle on `n_slices` batch slices of the decode workload, one slice
    at a time (32 heads x Lk keys each).  With `dev` the slices are cut from
    the workload's own device-drawn cache and copied to the host one by one
    (copy time excluded); otherwise each slice is drawn on the host with the
    workload's distribution.  Returns K/V GB/s and the extrapolated full run."""
    import torch
    from io_aware_exact_34_b200 import synth
    from oracle import oracle
    kv_bytes = 2.0 * wd.H * wd.Lk * wd.d * 2  # bf16 K and V of one slice
    dt = 0.0
    if dev is not None:
        q, k, v = synth.make_inputs(wd, device=dev)
        for b in range(n_slices):
            qs, ks, vs = (t[b:b + 1].cpu() for t in (q, k, v))
            t0 = time.perf_counter()
            oracle.attn(qs, ks, vs, wd.scale)
            dt += time.perf_counter() - t0
        del q, k, v
        torch.cuda.empty_cache()
    else:
        for b in range(n_slices):
            qs, ks, vs = synth.make_inputs(dataclasses.replace(wd, B=1), seed=wd.seed + 1000 + b)
            t0 = time.perf_counter()
            oracle.attn(qs, ks, vs, wd.scale)
            dt += time.perf_counter() - t0
    gbs = n_slices * kv_bytes / dt / 1e9
    return {"gbs": gbs, "slices": n_slices, "of_slices": wd.B, "seconds": dt,
            "extrapolated_full_run_s": wd.B * kv_bytes / (gbs * 1e9), "extrapolated": n_slices < wd.B,
            "source": "device cache, copied per slice" if dev is not None else "host draw per slice"}


def cpu_baseline(args, dev, budget_s=8.0):
    """The oracle, as it stands, on the host cores: the headline workload on
    whole heads for about `budget_s` seconds on all cores (the reported
    baseline) and on one head with one thread (per-core figure); the long
    prefill workloads on stratified row samples and the decode workload on
    batch slices, each with its full-run time extrapolated.  --cpu-full takes
    two full heads plus 4096 rows of every other head and every decode slice."""
    from io_aware_exact_34_b200 import synth
    from oracle import oracle
    oracle.build()
    w = synth.WORKLOADS[HEADLINE]
    q, k, v = synth.make_inputs(w)
    cores = oracle.num_threads()
    c = oracle.count_blocks(w.Lq, w.Lk, w.causal, w.window_left, w.window_right, 128, 128)
    head_flops = 4.0 * w.d * c["pairs"]
    heads, t0 = 0, time.perf_counter()
    for bh in range(w.B * w.H):
        b, h = divmod(bh, w.H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        oracle.attn(q[sl], k[sl], v[sl], w.scale, w.causal, w.window_left, w.window_right)
        heads += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    out = {"value": heads * head_flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
           "sample": f"{heads} of {w.B * w.H} (b,h) heads of {w.name}, every row, fp64, {dt:.1f} s on {cores} threads"}
    # per-core figure: one whole head on one thread
    oracle.set_num_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.attn(q[:1, :1], k[:1, :1], v[:1, :1], w.scale, w.causal, w.window_left, w.window_right)
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(cores)
    out["per_core"] = {"value": head_flops / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                       "sample": f"head (0,0) of {w.name}, every row, one thread, {dt1:.1f} s"}
    del q, k, v
    cfgs = {}
    for name in EXTRA:
        we = synth.WORKLOADS[name]
        if args.cpu_full:
            fh, nr = [(0, 0), (0, we.H - 1)], 4096
        else:
            fh, nr = ([] if we.Lq > 32768 else [(0, 0)]), 256
        cfgs[name] = cpu_sampled(we, fh, nr)
    wd = synth.WORKLOADS[DECODE]
    cfgs[DECODE] = cpu_decode_slices(wd, wd.B if args.cpu_full else 2, dev if args.cpu_full else None)
    out["configs"] = cfgs
    return out


def run_reference(args, world, rank):
    """The oracle timed on the host cores (the reference arm of this build)."""
    if rank != 0:
        return
    from io_aware_exact_34_b200 import synth
    from oracle import oracle
    oracle.build()
    w = synth.WORKLOADS[HEADLINE]
    q, k, v = synth.make_inputs(w)
    rows_per_step = 256
    g_rows = synth.sample_rows(w, n_random=0, seed=0, full_heads=[(w.B - 1, w.H - 1)]).numpy()
    g_rows = g_rows[g_rows[:, 0] == w.B - 1]
    g_rows = g_rows[g_rows[:, 1] == w.H - 1]

    # each step: 256 consecutive rows of the last head (every allowed key of each)
    def step(s):
        lo = (s * rows_per_step) % w.Lq
        rows = g_rows[lo:lo + rows_per_step]
        oracle.attn_rows(q, k, v, rows, w.scale, w.causal, w.window_left, w.window_right)
        return float(4.0 * w.d * allowed_keys(w, rows[:, 2]).sum())
    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    flops = 0.0
    for s in range(args.steps):
        flops += step(args.warmup + s)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s",
            "impl": "reference", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**w.describe(), "parallelism": "oracle on host cores"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{rows_per_step} consecutive query rows of head (b,h)=({w.B - 1},{w.H - 1}) per step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- GPU lines

def prefill_line(world, rank, dev, fl, peaks, peak_src, name, steps, warmup=3):
    """One dense prefill workload: TFLOP/s on in-mask FLOPs, roofline, tiles."""
    import torch
    from io_aware_exact_34_b200 import synth
    we = synth.WORKLOADS[name]
    f_e, c_e = prefill_flops(fl, we)
    eq, ek, ev = synth.make_inputs(we, device=dev, seed=replica_seed(we.seed, rank))
    eo = torch.empty_like(eq)
    el = torch.empty((we.B, we.H, we.Lq), dtype=torch.float32, device=dev)

    def estep():
        fl.attn_fwd(eq, ek, ev, o=eo, lse=el, scale=we.scale, causal=we.causal,
                    window_left=we.window_left, window_right=we.window_right)

    regions = []
    ems = timed_median(world, estep, steps, warmup, record=regions)
    sms = timed_sustained(world, estep, steps)
    tf = f_e / (ems * 1e-3) / 1e12
    line = {"value": world * tf, "unit": "TFLOP/s", "ms_per_step": ems, "steps": steps,
            "roofline": tensor_roofline(tf, peaks, peak_src, PREFILL_KERNEL, recorded_traffic(PREFILL_KERNEL, name)),
            "kv_tiles_visited_per_head": c_e["visited"], "kv_tiles_total_per_head": c_e["total"],
            "config": we.describe(), "gpu_launches": steps, "regions_ms": regions,
            "sustained": sustained_entry(world, sms, f_e, peaks)}
    if we.d < 128:
        line["exp_roofline"] = exp_roofline(tf, peaks, peak_src, we.d)
    del eq, ek, ev, eo, el
    torch.cuda.empty_cache()
    return line


def run_sweep(args, world, rank, dev, fl, peaks, peak_src):
    """The experiment matrix of the sliding-window prefill page, section 9.2:
    sequence length x window x batch, the tiled kernel with full attention
    against the same kernel with the bidirectional window |i - j| <= w (out-of-
    band tiles skipped).  One JSON line per point: times, TFLOP/s, tiles
    visited, peak device memory, and the measured speedup beside the page's
    n / (2w) estimate and the exact in-band pair ratio."""
    import torch
    from io_aware_exact_34_b200 import synth
    H, d = args.sweep_heads, 128
    for L in (4096, 8192, 16384, 32768):
        for B in (1, 2, 4, 8):
            torch.cuda.reset_peak_memory_stats()
            wf = synth.Workload(f"sweep_full_{B}x{L}", "prefill", B, H, L, L, d, "bf16", seed=9)
            q, k, v = synth.make_inputs(wf, device=dev, seed=replica_seed(9, rank))
            o = torch.empty_like(q)
            lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
            res = {}
            for wsz in (None, 2048, 1024, 512):
                wl = -1 if wsz is None else wsz

                def st():
                    fl.attn_fwd(q, k, v, o=o, lse=lse, window_left=wl, window_right=wl)

                steps = 3 if L * L * B >= 8 * 16384 * 16384 else 10
                ms = timed(world, st, steps, 3)
                c = fl.attn_count_blocks(L, L, False, wl, wl, 128, 128)
                fl_ = 4.0 * d * c["pairs"] * B * H
                res[wsz] = (ms, fl_, c)
            ms_full = res[None][0]
            for wsz in (None, 2048, 1024, 512):
                ms, fl_, c = res[wsz]
                tf = fl_ / (ms * 1e-3) / 1e12
                point = {"sweep": "p2_9.2", "seq": L, "batch": B, "heads": H, "d": d,
                         "window": "full" if wsz is None else wsz, "ms": ms, "tflops": tf,
                         "frac": tf / peaks["bf16_tflops"], "tiles_visited_per_head": c["visited"],
                         "tiles_total_per_head": c["total"],
                         "peak_mem_gb": torch.cuda.max_memory_allocated() / 1e9}
                if wsz is not None:
                    point.update(speedup_vs_full=ms_full / ms, page_estimate_n_over_2w=L / (2.0 * wsz),
                                 exact_pair_ratio=res[None][2]["pairs"] / c["pairs"])
                if rank == 0:
                    print(json.dumps(point), flush=True)
            del q, k, v, o, lse
            torch.cuda.empty_cache()


def run_ours(args, world, rank, local):
    import torch
    from io_aware_exact_34_b200 import fattn, synth
    peaks, peak_src = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    if args.sweep:
        run_sweep(args, world, rank, dev, fattn, peaks, peak_src)
        return

    # ---------------------------------------------------------------- headline prefill
    w = synth.WORKLOADS[HEADLINE]
    flops, counts = prefill_flops(fattn, w)
    q, k, v = synth.make_inputs(w, device=dev, seed=replica_seed(w.seed, rank))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Lq), dtype=torch.float32, device=dev)

    def step():
        fattn.attn_fwd(q, k, v, o=o, lse=lse, scale=w.scale, causal=w.causal,
                       window_left=w.window_left, window_right=w.window_right)

    ms, clocks, value, roofline, repeats, cold, sustained = float("nan"), None, None, None, None, None, None
    if not args.no_headline:
        def headline_regions():
            # the K-step region timed HEADLINE_REPEATS times; the median is the line's time
            out = [timed(world, step, args.steps, args.warmup)]
            for _ in range(HEADLINE_REPEATS - 1):
                out.append(timed(world, step, args.steps, 3))
            return out

        if args.no_clocks:
            reps = headline_regions()
            hs_ms = timed_sustained(world, step, args.steps, 1.0)
        else:
            with ClockSampler(local) as clk:
                reps = headline_regions()
                # keep the same work running for about a second so the sampler sees it
                t_end = time.perf_counter() + 1.0
                while time.perf_counter() < t_end:
                    for _ in range(20):
                        step()
                    torch.cuda.synchronize()
                # after a second of back-to-back work: the power-capped (sustained) regime
                hs_ms = timed(world, step, args.steps, 0) if SUSTAINED else None
            clocks = clk.summary()
        ms = statistics.median(reps)
        value = world * flops / (ms * 1e-3) / 1e12
        achieved = flops / (ms * 1e-3) / 1e12
        roofline = tensor_roofline(achieved, peaks, peak_src, PREFILL_KERNEL, recorded_traffic(PREFILL_KERNEL, w.name))
        repeats = {"n": len(reps), "steps_each": args.steps, "ms_per_step": reps, "median": ms,
                   "min": min(reps), "max": max(reps), "spread_pct": 100.0 * (max(reps) - min(reps)) / ms}
        sustained = sustained_entry(world, hs_ms, flops, peaks)
        if sustained:
            sustained["soak_s"] = 1.0
        # the same step with L2 flushed (a 256 MB write) before each launch
        flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
        cms = timed_cold_l2(world, step, args.steps, 3, flush)
        del flush
        ctf = flops / (cms * 1e-3) / 1e12
        cold = {"value": world * ctf, "unit": "TFLOP/s", "ms_per_step": cms, "steps": args.steps,
                "l2": "256 MB written before every step, outside its events",
                "roofline": tensor_roofline(ctf, peaks, peak_src, PREFILL_KERNEL, None)}

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e and not args.no_headline:
        # attn_fwd_host: pinned host Q, K, V in, host O and LSE out; the copies
        # of each chunk of heads overlap the kernels of the others
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        ws = torch.empty(fattn.attn_fwd_host_workspace_bytes(w.B, w.H, w.Lq, w.Lk, w.d), dtype=torch.uint8, device=dev)

        def e2e_step():
            fattn.attn_fwd_host(qh, kh, vh, o=oh, lse=lh, scale=w.scale, causal=w.causal,
                                window_left=w.window_left, window_right=w.window_right, workspace=ws)

        ms_e2e = timed(world, e2e_step, max(3, args.steps // 4), min(args.warmup, 3))
        e2e = {"value": world * flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": int(3 * q.numel() * q.element_size()),
               "d2h_bytes_per_step": int(o.numel() * o.element_size() + lse.numel() * 4)}
        del qh, kh, vh, oh, lh, ws

    # ---------------------------------------------------------------- backward (recomputation)
    bwd = None
    if not args.no_bwd:
        step()  # O and LSE of the forward, the backward's inputs
        dout = synth.random_dout(w.B, w.H, w.Lq, w.d, "bf16", seed=replica_seed(w.seed, rank), device=dev)
        gq, gk, gv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        gws = torch.empty(fattn.attn_bwd_workspace_bytes(w.B, w.H, w.Lq, w.d), dtype=torch.uint8, device=dev)

        def bstep():
            fattn.attn_bwd(q, k, v, o, dout, lse, scale=w.scale, causal=w.causal, window_left=w.window_left,
                           window_right=w.window_right, dq=gq, dk=gk, dv=gv, workspace=gws)

        bsteps = max(3, min(args.steps, 20))
        bregions = []
        bms = timed_median(world, bstep, bsteps, 3, record=bregions)
        bsms = timed_sustained(world, bstep, bsteps)
        bflops = 2.5 * flops  # five products per allowed pair instead of two
        tf = bflops / (bms * 1e-3) / 1e12
        rl = tensor_roofline(tf, peaks, peak_src, "attn_bwd_sm100_kernel",
                             recorded_traffic("attn_bwd_sm100_kernel", w.name))
        rl["kernels"] = ["bwd_prep_kernel", "attn_bwd_sm100_kernel", "bwd_dq_kernel"]
        bwd = {"metric": "attention bwd TFLOP/s (in-mask FLOPs: 10 d per allowed pair)", "value": world * tf,
               "unit": "TFLOP/s", "ms_per_step": bms, "steps": bsteps, "roofline": rl,
               "config": {**w.describe(), "pass": "backward with recomputation from LSE"},
               "gpu_launches": 3 * bsteps, "regions_ms": bregions,
               "sustained": sustained_entry(world, bsms, bflops, peaks)}
        del dout, gq, gk, gv, gws
        torch.cuda.empty_cache()

    # ---------------------------------------------------------------- FP8 forward
    fp8 = None
    if not args.no_fp8:
        q8, qs = fattn.attn_quantize_fp8(q)
        k8, ks = fattn.attn_quantize_fp8(k)
        vt8, vs = fattn.attn_quantize_fp8(v, transpose=True)
        o8 = torch.empty_like(o)

        def fstep():
            fattn.attn_fwd_fp8(q8, k8, vt8, qs, ks, vs, o=o8, lse=lse, scale=w.scale, causal=w.causal,
                               window_left=w.window_left, window_right=w.window_right)

        def qstep():
            fattn.attn_quantize_fp8(q, codes=q8, descale=qs)
            fattn.attn_quantize_fp8(k, codes=k8, descale=ks)
            fattn.attn_quantize_fp8(v, transpose=True, codes=vt8, descale=vs)

        fsteps = max(3, min(args.steps, 20))
        fregions = []
        fms = timed_median(world, fstep, fsteps, 3, record=fregions)
        fsms = timed_sustained(world, fstep, fsteps)
        qms = timed(world, qstep, 5, 3)
        tf = flops / (fms * 1e-3) / 1e12
        # nominal dense fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s) times the measured bf16 peak
        rl = tensor_roofline(tf, peaks, peak_src, PREFILL_KERNEL + "<128, false, true>",
                             recorded_traffic("attn_fwd_fp8", w.name), 2.0, " x 2 (nominal fp8/bf16 ratio)")
        fp8 = {"metric": "attention fwd TFLOP/s (in-mask FLOPs), e4m3 Q/K/V/P", "value": world * tf,
               "unit": "TFLOP/s", "ms_per_step": fms, "steps": fsteps, "roofline": rl,
               "exp_roofline": exp_roofline(tf, peaks, peak_src, w.d),
               "regions_ms": fregions, "sustained": sustained_entry(world, fsms, flops, peaks, 2.0),
               "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
               "quantize_ms_per_step": qms,
               "quantize_then_attend_tflops": world * flops / ((fms + qms) * 1e-3) / 1e12,
               "config": {**w.describe(), "dtype": "e4m3 (P e4m3, O bf16)"}, "gpu_launches": fsteps}
        del q8, k8, vt8, qs, ks, vs, o8
        torch.cuda.empty_cache()
    del q, k, v, o, lse
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- decode
    decode = None
    if not args.no_decode:
        wd = synth.WORKLOADS[DECODE]
        if args.decode_batch > 0:
            wd = dataclasses.replace(wd, B=args.decode_batch, name=f"{wd.name}_b{args.decode_batch}")
        dq, dk, dv = synth.make_inputs(wd, device=dev, seed=replica_seed(wd.seed, rank))
        do = torch.empty_like(dq)
        dl = torch.empty((wd.B, wd.H), dtype=torch.float32, device=dev)
        ws = torch.empty(fattn.attn_decode_workspace_bytes(wd.B, wd.H, wd.Lk, wd.d, wd.num_splits),
                         dtype=torch.uint8, device=dev)

        def dstep():
            fattn.attn_decode_splitkv(dq, dk, dv, o=do, lse=dl, scale=wd.scale, num_splits=wd.num_splits,
                                      workspace=ws)

        dsteps = max(5, min(args.steps, 40))
        dms = timed(world, dstep, dsteps, max(3, min(args.warmup, 5)))
        dbytes = (dk.numel() + dv.numel() + dq.numel() + do.numel()) * 2 + dl.numel() * 4
        gbs = dbytes / (dms * 1e-3) / 1e9
        decode = {"metric": "decode HBM GB/s", "value": world * gbs, "unit": "GB/s", "ms_per_step": dms,
                  "steps": dsteps, "config": wd.describe(),
                  "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": gbs / peaks["hbm_gbs"], "traffic": recorded_traffic("decode_split_kernel", wd.name),
                               "peak_source": f"{peak_src} copy bandwidth",
                               "kernels": ["decode_split_kernel", "decode_merge_kernel"]},
                  "bytes_per_step": int(dbytes), "gpu_launches": 2 * dsteps}
        del dq, dk, dv, do, ws
        torch.cuda.empty_cache()

    # ---------------------------------------------------------------- paged-KV decode
    decode_paged = None
    if not args.no_decode and not args.no_extra:
        wd = dataclasses.replace(synth.WORKLOADS[DECODE], name=synth.WORKLOADS[DECODE].name + "_paged")
        if args.decode_batch > 0:
            wd = dataclasses.replace(wd, B=args.decode_batch, name=f"{wd.name}_b{args.decode_batch}")
        pq, kp, vp, table, seqlens = synth.make_paged_inputs(wd.B, wd.H, wd.Lk, wd.d, PAGE_SIZE,
                                                             seed=replica_seed(7, rank), device=dev)
        po = torch.empty_like(pq)
        pl = torch.empty((wd.B, wd.H), dtype=torch.float32, device=dev)
        pws = torch.empty(fattn.attn_decode_workspace_bytes(wd.B, wd.H, wd.Lk, wd.d, wd.num_splits),
                          dtype=torch.uint8, device=dev)

        def pstep():
            fattn.attn_decode_paged(pq, kp, vp, table, seqlens, o=po, lse=pl, scale=wd.scale,
                                    num_splits=wd.num_splits, workspace=pws)

        psteps = max(5, min(args.steps, 20))
        pms = timed(world, pstep, psteps, 3)
        pbytes = (kp.numel() + vp.numel() + pq.numel() + po.numel()) * 2 + pl.numel() * 4 + table.numel() * 4
        gbs = pbytes / (pms * 1e-3) / 1e9
        decode_paged = {"metric": "decode HBM GB/s", "value": world * gbs, "unit": "GB/s", "ms_per_step": pms,
                        "steps": psteps,
                        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": gbs / peaks["hbm_gbs"],
                                     "traffic": recorded_traffic("decode_split_kernel", wd.name),
                                     "peak_source": f"{peak_src} copy bandwidth",
                                     "kernels": ["decode_split_kernel", "decode_merge_kernel"]},
                        "config": {**wd.describe(), "workload": wd.name, "page_size": PAGE_SIZE,
                                   "layout": "pages [num_pages, page_size, H, d], random block table"},
                        "gpu_launches": 2 * psteps}
        del pq, kp, vp, table, po, pws
        torch.cuda.empty_cache()

    # ---------------------------------------------------------------- other prefill workloads
    extra = {}
    if not args.no_extra and not args.no_d64:
        extra[HEADLINE_D64] = prefill_line(world, rank, dev, fattn, peaks, peak_src, HEADLINE_D64,
                                           max(3, min(args.steps, 20)))
        extra[WINDOW_D64] = prefill_line(world, rank, dev, fattn, peaks, peak_src, WINDOW_D64,
                                         max(3, min(args.steps, 10)))
    if not args.no_extra and not args.no_windows:
        for name in EXTRA:
            extra[name] = prefill_line(world, rank, dev, fattn, peaks, peak_src, name, max(3, min(args.steps, 10)))

    # ---------------------------------------------------------------- packed variable-length prefill
    if not args.no_extra and not args.no_varlen:
        lens = synth.varlen_lengths(VARLEN_SEQS, VARLEN_MIN, VARLEN_MAX, seed=replica_seed(6, rank))
        vq, vk, vv, cuq, cuk = synth.make_varlen_inputs(lens, lens, VARLEN_H, 128, seed=replica_seed(6, rank), device=dev)
        vo = torch.empty_like(vq)
        vl = torch.empty((VARLEN_H, vq.shape[0]), dtype=torch.float32, device=dev)
        f_v = sum(4.0 * 128 * fattn.attn_count_blocks(L, L, True, -1, -1, 128, 128)["pairs"] * VARLEN_H for L in lens)

        def vstep():
            fattn.attn_fwd_varlen(vq, vk, vv, cuq, cuk, max(lens), o=vo, lse=vl, causal=True)

        vsteps = max(3, min(args.steps, 10))
        vregions = []
        vms = timed_median(world, vstep, vsteps, 3, record=vregions)
        vsms = timed_sustained(world, vstep, vsteps)
        tf = f_v / (vms * 1e-3) / 1e12
        extra["varlen_causal_32seq"] = {
            "value": world * tf, "unit": "TFLOP/s", "ms_per_step": vms, "steps": vsteps,
            "regions_ms": vregions, "sustained": sustained_entry(world, vsms, f_v, peaks),
            "roofline": tensor_roofline(tf, peaks, peak_src, PREFILL_KERNEL + "<128, true, false>",
                                        recorded_traffic(PREFILL_KERNEL, "varlen_causal_32seq")),
            "config": {"workload": "varlen_causal_32seq", "num_seqs": VARLEN_SEQS,
                       "seqlen_range": [VARLEN_MIN, VARLEN_MAX], "total_tokens": int(sum(lens)),
                       "H": VARLEN_H, "d": 128, "causal": True, "layout": "packed [total, H, d]"},
            "gpu_launches": vsteps}
        del vq, vk, vv, vo, vl
        torch.cuda.empty_cache()

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, dev)

    if rank == 0:
        def tf_frac(x):
            return None if x is None else [r4(x["value"]), r4(x["roofline"]["frac"])]

        summary = {"headline": tf_frac({"value": value, "roofline": roofline}) if value is not None else None,
                   "headline_spread_pct": r4(repeats["spread_pct"]) if repeats else None,
                   "cold_l2": tf_frac(cold), "e2e_tflops": r4(e2e["value"]) if e2e else None,
                   "bwd": tf_frac(bwd), "fp8": tf_frac(fp8),
                   "fp8_quantize_ms": r4(fp8["quantize_ms_per_step"]) if fp8 else None,
                   "decode_gbs": tf_frac(decode), "decode_paged_gbs": tf_frac(decode_paged),
                   "extra": {n: tf_frac(x) for n, x in extra.items()},
                   "exp_frac": {n: r4(x["exp_roofline"]["frac"])
                                for n, x in [("fp8", fp8), *extra.items()] if x and "exp_roofline" in x},
                   "sustained": {n: [r4(x["sustained"]["value"]), r4(x["sustained"]["frac"])]
                                 for n, x in [("headline", {"sustained": sustained}), ("bwd", bwd), ("fp8", fp8),
                                              *extra.items()] if x and x.get("sustained")}}
        if cpu:
            summary["cpu"] = {"all_cores_tflops": r4(cpu["value"]), "one_core_tflops": r4(cpu["per_core"]["value"]),
                              "cores": cpu["cores"]}
            for n, x in cpu["configs"].items():
                summary["cpu"][n] = ({"gbs": r4(x["gbs"]), "full_s_extrap": r4(x["extrapolated_full_run_s"])}
                                     if "gbs" in x else
                                     {"tflops": r4(x["tflops"]), "full_s_extrap": r4(x["extrapolated_full_run_s"])})
        line = {"metric": METRIC,
                "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {**w.describe(), "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                           "l2": "inputs 201 MB (Q+K+V) > 126 MB L2, no flush (cold_l2: flushed)",
                           "kv_tiles_visited_per_head": counts["visited"],
                           "kv_tiles_total_per_head": counts["total"]},
                "roofline": roofline, "e2e": e2e, "gpu_launches": args.steps, "repeats": repeats,
                "sustained": sustained,
                "cold_l2": cold, "clocks": clocks, "decode": decode, "decode_paged": decode_paged,
                "bwd": bwd, "fp8": fp8, "extra": extra, "cpu_baseline": cpu,
                "summary": summary}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-headline", action="store_true", help="skip the headline prefill (profiling runs)")
    ap.add_argument("--decode-batch", type=int, default=0, help="override the decode batch (profiling runs)")
    ap.add_argument("--no-clocks", action="store_true", help="no nvidia-smi sampling or soak (profiling runs)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-windows", action="store_true", help="skip the window and 64K lines (keeps varlen)")
    ap.add_argument("--no-varlen", action="store_true", help="skip the packed varlen line")
    ap.add_argument("--no-d64", action="store_true", help="skip the d = 64 prefill lines")
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-fp8", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sustained", action="store_true", help="skip the sustained regions (profiling runs)")
    ap.add_argument("--regions", type=int, default=3, help="burst regions per secondary line (median taken)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-full", action="store_true",
                    help="CPU baseline on two full heads + 4096 rows of every other head, and every decode slice")
    ap.add_argument("--sweep", action="store_true",
                    help="sequence x window x batch matrix of the sliding-window page (one JSON line per point)")
    ap.add_argument("--sweep-heads", type=int, default=32)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    global REGIONS, SUSTAINED
    REGIONS = max(1, args.regions)
    SUSTAINED = not args.no_sustained
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup(args)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
