"""Benchmark of the packed variable-length attention forward on B200.

Prints ONE JSON line (rank 0).  Metric: prefill TFLOP/s of the varlen forward
(algorithmic FLOPs = 4 * visible (q, k) pairs * D * H) on the 16-sequence
non-causal MHA workload (q = k lengths uniform-int in [64, 2048], H = H_kv =
16, D = 128), with the decode-shape HBM GB/s (128 sequences of one query,
k lengths uniform-int in [1024, 32768], H = 32, H_kv = 8, D = 128) reported
beside it under "decode", the chunked-prefill workload under
"chunked_prefill", the same headline workload in FP8 (E4M3 inputs and
output with per-tensor scales, varlen_attention_fwd_fp8) under "fp8" and its
backward pass (varlen_attention_bwd) under "backward".  A step
is one call of the C ABI on one batch: schedule build + prefill kernel
(decode: split + combine kernels).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME]

Under torchrun each rank runs its own batch (seed + rank): no collective
touches the data path (weak scaling); the elapsed time is the max over ranks.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from variable_length_flash_varlen_b200 import accounting, binding, workloads  # noqa: E402

METRIC = "varlen FA fwd TFLOP/s + % BF16 TC peak; decode-shape HBM GB/s + % peak"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers --

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Sources each kernel is compiled from (the launch code in varlen_attn.cu
# included), so a recorded traffic figure goes stale only when its own kernel
# changes.
KERNEL_SOURCES = {
    "prefill_fwd_kernel": ("prefill_sm100.cuh", "f32x2.cuh", "schedule.cuh", "ptx.cuh", "status.cuh",
                           "varlen_attn.cu"),
    "decode_stream_kernel": ("decode.cuh", "schedule.cuh", "ptx.cuh", "status.cuh", "varlen_attn.cu"),
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "variable_length_flash_varlen_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches these sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    e = rec.get(kernel, {}).get(workload)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        if self.index is None:
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = os.environ.get("BENCH_DIST_BACKEND") or ("nccl" if torch.cuda.is_available() else "gloo")
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------- CPU oracle --

def oracle_sample(wl, q, k, v, target_s: float, seed: int = 0):
    """Time the fp64 oracle on a random sample of (token, head) rows of `wl`.

    Returns (algorithmic FLOPs of the sample, seconds, threads, rows).
    """
    import numpy as np
    from oracle import oracle
    oracle.build()
    threads = oracle.default_threads()
    rng = np.random.default_rng(seed)
    total_rows = wl.total_q * wl.H
    lens_q = np.array(wl.lengths_q)
    lens_k = np.array(wl.lengths_k)
    cu_q = np.array(wl.cu_q)

    def flops_of(rows):
        b = np.searchsorted(cu_q, rows[:, 0], side="right") - 1
        i = rows[:, 0] - cu_q[b]
        Lq, Lk = lens_q[b], lens_k[b]
        delta = Lk - Lq
        hi = Lk - 1
        if wl.causal or wl.window > 0:
            hi = np.minimum(hi, i + delta)
        lo = np.maximum(0, i + delta - wl.window + 1) if wl.window > 0 else np.zeros_like(i)
        vis = np.maximum(0, hi - lo + 1)
        return float(4.0 * vis.sum() * wl.D)

    def run(n):
        rows = np.stack([rng.integers(0, wl.total_q, n), rng.integers(0, wl.H, n)], axis=1)
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D, wl.causal,
                              wl.window, rows=rows, nthreads=threads)
        return flops_of(rows), time.perf_counter() - t0

    n = max(threads * 4, 256)
    f, t = run(n)
    while t < 0.5 and n < total_rows:
        n = min(total_rows, n * 4)
        f, t = run(n)
    if t < target_s and n < total_rows:
        n = int(min(total_rows, n * target_s / max(t, 1e-3)))
        f, t = run(n)
    return f, t, threads, n


# ------------------------------------------------------------------- arms --

def run_reference(args, world, rank):
    """The oracle as the reference arm: bounded samples of the workload on host cores."""
    if rank != 0:
        return None
    wl = workloads.named(args.workload)
    q, k, v = workloads.make_qkv(wl)
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(wl, q, k, v, target_s=min(per_step, 2.0))
    flops, secs, rows = 0.0, 0.0, 0
    threads = 1
    for s in range(args.steps):
        f, t, threads, n = oracle_sample(wl, q, k, v, target_s=per_step, seed=s + 1)
        flops += f
        secs += t
        rows += n
    value = flops / secs / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, **wl.describe(), "parallelism": f"dp{args.gpus}"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} random (token, head) rows over {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def time_device_steps(fn, steps, warmup, flush_buf, world, stream):
    """Per-step CUDA-event time of fn() (L2 flushed before each step, outside the events)."""
    for _ in range(warmup):
        flush_buf.zero_()
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    outer0, outer1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    outer0.record(stream)
    for i in range(steps):
        flush_buf.zero_()
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    outer1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return step_ms, outer0.elapsed_time(outer1)


def run_profile_target(args, local):
    """Run only the prefill, the FP8 prefill or the decode call (warm-up + steps) for an ncu capture."""
    dev = torch.device("cuda", local)
    binding.load()
    name = "decode" if args.only == "decode" else args.workload
    wl = workloads.named(name, scale=args.scale)
    if args.only == "fp8":
        q8, k8, v8, sc = workloads.make_qkv_fp8(wl)
        d8 = [t.to(dev) for t in (q8, k8, v8)]
        cq = torch.tensor(wl.cu_q, dtype=torch.int32, device=dev)
        ck = torch.tensor(wl.cu_k, dtype=torch.int32, device=dev)
        out8 = torch.empty_like(d8[0])
        lse8 = torch.empty(wl.total_q, wl.H, dtype=torch.float32, device=dev)
        for _ in range(args.warmup + args.steps):
            binding.varlen_attention_fwd_fp8(*d8, cq, ck, wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q,
                                             wl.max_seqlen_k, wl.D, wl.causal, wl.window,
                                             sc["q_scale"], sc["k_scale"], sc["v_scale"],
                                             sc["o_scale"], out=out8, lse=lse8)
        torch.cuda.synchronize()
        if binding.device_status() != 0:
            raise SystemExit("device status word raised")
        return
    q, k, v = workloads.make_qkv(wl)
    dq, dk, dv = q.to(dev), k.to(dev), v.to(dev)
    cq = torch.tensor(wl.cu_q, dtype=torch.int32, device=dev)
    ck = torch.tensor(wl.cu_k, dtype=torch.int32, device=dev)
    out = torch.empty_like(dq)
    lse = torch.empty(wl.total_q, wl.H, dtype=torch.float32, device=dev)
    if args.only == "bwd":
        binding.varlen_attention_fwd(dq, dk, dv, cq, ck, wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q,
                                     wl.max_seqlen_k, wl.D, wl.causal, wl.window, out=out, lse=lse)
        gen = torch.Generator().manual_seed(workloads.WORKLOAD_SEEDS[args.workload] + 7)
        ddo = torch.randn(wl.total_q, wl.H, wl.D, generator=gen).to(torch.bfloat16).to(dev)
        for _ in range(args.warmup + args.steps):
            binding.varlen_attention_bwd(ddo, dq, dk, dv, out, lse, cq, ck, wl.batch, wl.H, wl.H_kv,
                                         wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal, wl.window)
        torch.cuda.synchronize()
        if binding.device_status() != 0:
            raise SystemExit("device status word raised")
        return
    for _ in range(args.warmup + args.steps):
        binding.varlen_attention_fwd(dq, dk, dv, cq, ck, wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q,
                                     wl.max_seqlen_k, wl.D, wl.causal, wl.window, out=out, lse=lse)
    torch.cuda.synchronize()
    if binding.device_status() != 0:
        raise SystemExit("device status word raised")


def run_ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_kind = load_peaks()
    binding.load()

    # ---- prefill workload (the headline)
    wl = workloads.named(args.workload, seed=workloads.WORKLOAD_SEEDS[args.workload] + rank)
    q, k, v = workloads.make_qkv(wl)
    dq, dk, dv = q.to(dev), k.to(dev), v.to(dev)
    cq = torch.tensor(wl.cu_q, dtype=torch.int32, device=dev)
    ck = torch.tensor(wl.cu_k, dtype=torch.int32, device=dev)
    out = torch.empty_like(dq)
    lse = torch.empty(wl.total_q, wl.H, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flops = accounting.attention_flops(wl)

    def step():
        binding.varlen_attention_fwd(dq, dk, dv, cq, ck, wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q,
                                     wl.max_seqlen_k, wl.D, wl.causal, wl.window, out=out, lse=lse)

    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_index = int(visible.split(",")[local]) if visible and visible.split(",")[local].isdigit() else local
    # clocks are sampled across all timed loops (prefill, decode, chunked prefill, end to end)
    clk = ClockSampler(smi_index if not args.no_clock_sampler else None).__enter__()
    step_ms, outer_ms = time_device_steps(step, args.steps, args.warmup, flush, world, stream)
    t_local = sum(step_ms) / 1e3
    t_max = max_over_ranks(t_local, world)
    total_flops = sum_over_ranks(flops * args.steps, world)
    value = total_flops / t_max / 1e12
    per_launch_s = t_local / args.steps
    achieved = flops / per_launch_s / 1e12
    peak = peaks["bf16_tflops"]

    # ---- decode workload (the HBM half of the metric)
    dwl = workloads.named("decode", seed=workloads.WORKLOAD_SEEDS["decode"] + rank)
    qd, kd, vd = workloads.make_qkv(dwl)
    dqd, dkd, dvd = qd.to(dev), kd.to(dev), vd.to(dev)
    cqd = torch.tensor(dwl.cu_q, dtype=torch.int32, device=dev)
    ckd = torch.tensor(dwl.cu_k, dtype=torch.int32, device=dev)
    outd = torch.empty_like(dqd)
    lsed = torch.empty(dwl.total_q, dwl.H, dtype=torch.float32, device=dev)

    def dstep():
        binding.varlen_attention_fwd(dqd, dkd, dvd, cqd, ckd, dwl.batch, dwl.H, dwl.H_kv,
                                     dwl.max_seqlen_q, dwl.max_seqlen_k, dwl.D, dwl.causal,
                                     dwl.window, out=outd, lse=lsed)

    d_ms, _ = time_device_steps(dstep, args.steps, args.warmup, flush, world, stream)
    d_local = sum(d_ms) / 1e3
    d_max = max_over_ranks(d_local, world)
    dbytes = accounting.decode_bytes(dwl)
    d_value = sum_over_ranks(dbytes * args.steps, world) / d_max / 1e9
    del dqd, dkd, dvd, outd, lsed

    # ---- chunked prefill: new query chunks after cached prefixes (L_q < L_k, causal)
    cwl = workloads.named("chunked_prefill", seed=workloads.WORKLOAD_SEEDS["chunked_prefill"] + rank)
    qc, kc, vc = workloads.make_qkv(cwl)
    dqc, dkc, dvc = qc.to(dev), kc.to(dev), vc.to(dev)
    cqc = torch.tensor(cwl.cu_q, dtype=torch.int32, device=dev)
    ckc = torch.tensor(cwl.cu_k, dtype=torch.int32, device=dev)
    outc = torch.empty_like(dqc)
    lsec = torch.empty(cwl.total_q, cwl.H, dtype=torch.float32, device=dev)

    def cstep():
        binding.varlen_attention_fwd(dqc, dkc, dvc, cqc, ckc, cwl.batch, cwl.H, cwl.H_kv,
                                     cwl.max_seqlen_q, cwl.max_seqlen_k, cwl.D, cwl.causal,
                                     cwl.window, out=outc, lse=lsec)

    c_ms, _ = time_device_steps(cstep, args.steps, args.warmup, flush, world, stream)
    c_max = max_over_ranks(sum(c_ms) / 1e3, world)
    cflops = accounting.attention_flops(cwl)
    c_value = sum_over_ranks(cflops * args.steps, world) / c_max / 1e12
    del dqc, dkc, dvc, outc, lsec, qc, kc, vc

    # ---- FP8 (E4M3) forward on the headline workload (flash_attention_fwd_fp8 semantics)
    fq, fk, fv, fsc = workloads.make_qkv_fp8(wl)
    dfq, dfk, dfv = fq.to(dev), fk.to(dev), fv.to(dev)
    fout = torch.empty_like(dfq)
    flse = torch.empty(wl.total_q, wl.H, dtype=torch.float32, device=dev)

    def fstep():
        binding.varlen_attention_fwd_fp8(dfq, dfk, dfv, cq, ck, wl.batch, wl.H, wl.H_kv,
                                         wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal,
                                         wl.window, fsc["q_scale"], fsc["k_scale"], fsc["v_scale"],
                                         fsc["o_scale"], out=fout, lse=flse)

    f_ms, _ = time_device_steps(fstep, args.steps, args.warmup, flush, world, stream)
    f_max = max_over_ranks(sum(f_ms) / 1e3, world)
    f_value = total_flops / f_max / 1e12
    # E4M3 dense tensor peak: the measured bf16 peak times the nominal fp8 / bf16 ratio (4.5 / 2.25)
    fp8_peak = peak * 2.0
    del dfq, dfk, dfv, fout, flse, fq, fk, fv

    # ---- backward pass on the headline workload (dq, dk, dv from the forward's out and lse)
    gen = torch.Generator().manual_seed(workloads.WORKLOAD_SEEDS[args.workload] + 7 + rank)
    ddo = torch.randn(wl.total_q, wl.H, wl.D, generator=gen).to(torch.bfloat16).to(dev)
    binding.varlen_attention_fwd(dq, dk, dv, cq, ck, wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q,
                                 wl.max_seqlen_k, wl.D, wl.causal, wl.window, out=out, lse=lse)
    gq, gk, gv = torch.empty_like(dq), torch.empty_like(dk), torch.empty_like(dv)

    def bstep():
        binding.varlen_attention_bwd(ddo, dq, dk, dv, out, lse, cq, ck, wl.batch, wl.H, wl.H_kv,
                                     wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal, wl.window,
                                     dq=gq, dk=gk, dv=gv)

    b_ms, _ = time_device_steps(bstep, args.steps, args.warmup, flush, world, stream)
    b_max = max_over_ranks(sum(b_ms) / 1e3, world)
    bflops = accounting.backward_flops(wl)
    b_value = sum_over_ranks(bflops * args.steps, world) / b_max / 1e12
    del ddo, gq, gk, gv

    # ---- end to end through the host-buffer entry point (pinned memory)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    cqh = torch.tensor(wl.cu_q, dtype=torch.int32)
    ckh = torch.tensor(wl.cu_k, dtype=torch.int32)
    outh = torch.empty_like(q).pin_memory()
    lseh = torch.empty(wl.total_q, wl.H, dtype=torch.float32).pin_memory()

    def estep():
        binding.varlen_attention_fwd_host(qh, kh, vh, cqh, ckh, wl.batch, wl.H, wl.H_kv,
                                          wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal,
                                          wl.window, outh, lseh)

    e_ms, _ = time_device_steps(estep, args.steps, args.warmup, flush, world, stream)
    clk.__exit__(None, None, None)
    e_max = max_over_ranks(sum(e_ms) / 1e3, world)
    e_value = total_flops / e_max / 1e12
    h2d = (q.numel() + k.numel() + v.numel()) * 2 + (len(wl.cu_q) + len(wl.cu_k)) * 4
    d2h = out.numel() * 2 + lse.numel() * 4

    if rank != 0:
        return None

    # ---- CPU oracle baseline on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not args.skip_cpu_baseline:
        f, t, threads, n = oracle_sample(wl, q, k, v, target_s=args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} random (token, head) rows of the same workload, {t:.1f} s"}

    clocks = clk.summary()
    d_frac = d_value / (peaks["hbm_gbs"] * world)
    return {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_max / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, **wl.describe(), "parallelism": f"dp{world}",
                   "l2": "256 MiB buffer written before every step, outside the step events",
                   "flops_per_step_per_gpu": flops},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_kind": f"{peak_kind} bf16 burst",
                     "kernel": "prefill_fwd_kernel<128> (+ schedule build, same call)",
                     "traffic": recorded_traffic("prefill_fwd_kernel", args.workload)},
        "decode": {"workload": "decode", **dwl.describe(), "value": d_value, "unit": "GB/s",
                   "ms_per_step": d_max / args.steps * 1e3, "bytes_per_step": dbytes,
                   "roofline": {"bound": "hbm", "achieved": d_value / world,
                                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": d_frac,
                                "peak_kind": f"{peak_kind} copy",
                                "kernel": "decode_stream_kernel<128> (+ combine and counter reset, same call)",
                                "traffic": recorded_traffic("decode_stream_kernel", "decode")},
                   "gpu_launches": 2 * args.steps},
        "chunked_prefill": {**cwl.describe(), "value": c_value, "unit": "TFLOP/s",
                            "ms_per_step": c_max / args.steps * 1e3, "flops_per_step_per_gpu": cflops,
                            "roofline": {"bound": "tensor", "achieved": c_value / world, "peak": peak,
                                         "unit": "TFLOP/s", "frac": c_value / world / peak,
                                         "peak_kind": f"{peak_kind} bf16 burst"},
                            "gpu_launches": 2 * args.steps},
        "fp8": {"workload": args.workload, "entry": "varlen_attention_fwd_fp8", "dtype": "e4m3",
                "scales": fsc, "value": f_value, "unit": "TFLOP/s",
                "ms_per_step": f_max / args.steps * 1e3,
                "roofline": {"bound": "tensor", "achieved": f_value / world, "peak": fp8_peak,
                             "unit": "TFLOP/s", "frac": f_value / world / fp8_peak,
                             "peak_kind": f"{peak_kind} bf16 burst x 2 (nominal e4m3 / bf16 ratio)",
                             "kernel": "prefill_fwd_kernel<128, E4M3> (+ schedule build, same call)"},
                "gpu_launches": 2 * args.steps},
        "backward": {"workload": args.workload, "entry": "varlen_attention_bwd", "value": b_value,
                     "unit": "TFLOP/s", "ms_per_step": b_max / args.steps * 1e3,
                     "flops_per_step_per_gpu": bflops,
                     "roofline": {"bound": "tensor", "achieved": b_value / world, "peak": peak,
                                  "unit": "TFLOP/s", "frac": b_value / world / peak,
                                  "peak_kind": f"{peak_kind} bf16 burst",
                                  "kernel": "bwd_delta + bwd_dkdv + bwd_dq (same call)"},
                     "gpu_launches": 3 * args.steps},
        "e2e": {"value": e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "outer_ms_with_flush": outer_ms,
        "step_ms": [round(x, 4) for x in step_ms],
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mha_noncausal", choices=list(workloads.WORKLOAD_SEEDS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--no-clock-sampler", action="store_true")
    ap.add_argument("--scale", type=float, default=1.0,
                    help="shrink every sequence length (profiling captures of a small case)")
    ap.add_argument("--only", choices=["all", "prefill", "fp8", "bwd", "decode"], default="all",
                    help="profiling: run only one half of the step (no JSON line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup()
    if args.only != "all":
        run_profile_target(args, local)
        res = None
    elif args.impl == "reference":
        res = run_reference(args, world, rank)
    else:
        if not torch.cuda.is_available():
            raise SystemExit("the CUDA path needs a GPU; there is no CPU fallback")
        res = run_ours(args, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
