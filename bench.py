"""Benchmark of the packed variable-length attention forward on B200.

Prints ONE JSON line (rank 0).  Metric: prefill TFLOP/s of the varlen forward
(algorithmic FLOPs = 4 * visible (q, k) pairs * D * H) with its fraction of
the bf16 tensor peak, headlined on the largest configuration, the sliding
window (4 sequences of 32768 tokens, window 4096, causal, H=32, H_kv=8,
D=128, 8.25 TFLOP per call).  Beside it: every other prefill configuration
(the worked example, the 16-sequence non-causal MHA workload, the GQA causal
workload) under "prefill_configs", the decode-shape HBM GB/s (128 sequences
of one query, k lengths uniform-int in [1024, 32768], H=32, H_kv=8, D=128)
under "decode", the chunked-prefill workload under "chunked_prefill", the MHA
workload in FP8 (E4M3 inputs and output with per-tensor scales,
varlen_attention_fwd_fp8) under "fp8", the backward pass (varlen_attention_bwd)
on the MHA and GQA workloads under "backward", and the headline end to end
through the host-buffer entry point under "e2e".  A step is one call of the C
ABI on one batch: schedule build + prefill kernel (decode: split + combine
kernels).

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
# every prefill configuration of the metric, each timed in its own loop; the
# headline (--workload) is the largest one that fits one GPU
PREFILL_CONFIGS = ("worked_example", "mha_noncausal", "gqa_causal", "sliding_window")
BACKWARD_CONFIGS = ("mha_noncausal", "gqa_causal")
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


# Device sources each kernel is compiled from (its block size, shared memory
# and launch shape are constants of these headers; the grid is one CTA per SM),
# so a recorded traffic figure goes stale only when its own kernel changes.
KERNEL_SOURCES = {
    "prefill_fwd_kernel": ("prefill_sm100.cuh", "f32x2.cuh", "schedule.cuh", "ptx.cuh", "status.cuh"),
    "decode_stream_kernel": ("decode.cuh", "schedule.cuh", "ptx.cuh", "status.cuh"),
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
    """Per-step CUDA-event time of fn() (L2 flushed before each step, outside the
    events), the whole loop's time, and the library kernels launched in it."""
    for _ in range(warmup):
        flush_buf.zero_()
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    outer0, outer1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = binding.launch_count()
    outer0.record(stream)
    for i in range(steps):
        flush_buf.zero_()
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    outer1.record(stream)
    launches = binding.launch_count() - launches0
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return step_ms, outer0.elapsed_time(outer1), launches


def run_profile_target(args, local):
    """Run only the prefill, the FP8 prefill or the decode call (warm-up + steps) for an ncu capture."""
    dev = torch.device("cuda", local)
    binding.load()
    name = "decode" if args.only == "decode" else args.workload
    wl = workloads.named(name, scale=args.scale)
    if args.first_seqs > 0:
        # the first N sequences alone (a smaller capture whose work, and traffic,
        # is the full workload's share of those sequences)
        n = args.first_seqs
        wl = workloads.custom(wl.lengths_q[:n], wl.lengths_k[:n], wl.H, wl.H_kv, wl.D, wl.causal,
                              wl.window, wl.seed, name=wl.name)
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


def _inputs_on(wl, dev):
    q, k, v = workloads.make_qkv(wl)
    cq = torch.tensor(wl.cu_q, dtype=torch.int32, device=dev)
    ck = torch.tensor(wl.cu_k, dtype=torch.int32, device=dev)
    return (q, k, v), (q.to(dev), k.to(dev), v.to(dev), cq, ck)


def _fwd_call(wl, d, out, lse):
    dq, dk, dv, cq, ck = d
    return lambda: binding.varlen_attention_fwd(dq, dk, dv, cq, ck, wl.batch, wl.H, wl.H_kv,
                                                wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal,
                                                wl.window, out=out, lse=lse)


def _tensor_roofline(achieved, peak, peak_kind, **extra):
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "peak_kind": peak_kind, **extra}


def run_ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_kind = load_peaks()
    peak = peaks["bf16_tflops"]
    pk = f"{peak_kind} bf16 burst"
    binding.load()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    seed = lambda name: workloads.WORKLOAD_SEEDS[name] + rank  # noqa: E731

    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_index = int(visible.split(",")[local]) if visible and visible.split(",")[local].isdigit() else local
    # clocks are sampled across all timed loops
    clk = ClockSampler(smi_index if not args.no_clock_sampler else None).__enter__()

    launches = {}

    def timed(fn, leg):
        ms, _, n = time_device_steps(fn, args.steps, args.warmup, flush, world, stream)
        launches[leg] = n
        local_s = sum(ms) / 1e3
        return ms, local_s, max_over_ranks(local_s, world)

    def prefill_leg(name):
        wl = workloads.named(name, seed=seed(name))
        host, d = _inputs_on(wl, dev)
        out = torch.empty_like(d[0])
        lse = torch.empty(wl.total_q, wl.H, dtype=torch.float32, device=dev)
        flops = accounting.attention_flops(wl)
        ms, local_s, max_s = timed(_fwd_call(wl, d, out, lse), name)
        value = sum_over_ranks(flops * args.steps, world) / max_s / 1e12
        achieved = flops / (local_s / args.steps) / 1e12
        return wl, host, d, (out, lse), {
            "workload": name, **wl.describe(), "value": value, "unit": "TFLOP/s",
            "ms_per_step": max_s / args.steps * 1e3, "flops_per_step_per_gpu": flops,
            "roofline": _tensor_roofline(achieved, peak, pk,
                                         kernel=f"prefill_fwd_kernel<{wl.D}> (+ schedule build, same call)",
                                         traffic=recorded_traffic("prefill_fwd_kernel", name)),
            "gpu_launches": launches[name]}, ms

    # ---- the headline: prefill TFLOP/s on the largest configuration (sliding window)
    wl, host, d, (out, lse), head, step_ms = prefill_leg(args.workload)
    q, k, v = host

    # ---- the other prefill configurations, each its own timed loop
    prefill_configs = {}
    for name in PREFILL_CONFIGS:
        if name != args.workload:
            r = prefill_leg(name)
            prefill_configs[name] = r[4]
            del r

    # ---- decode workload (the HBM half of the metric)
    dwl = workloads.named("decode", seed=seed("decode"))
    _, dd = _inputs_on(dwl, dev)
    outd = torch.empty_like(dd[0])
    lsed = torch.empty(dwl.total_q, dwl.H, dtype=torch.float32, device=dev)
    _, d_local, d_max = timed(_fwd_call(dwl, dd, outd, lsed), "decode")
    dbytes = accounting.decode_bytes(dwl)
    d_value = sum_over_ranks(dbytes * args.steps, world) / d_max / 1e9
    del dd, outd, lsed

    # ---- chunked prefill: new query chunks after cached prefixes (L_q < L_k, causal)
    chunked = prefill_leg("chunked_prefill")[4]

    # ---- FP8 (E4M3) forward on the MHA workload (flash_attention_fwd_fp8 semantics)
    fwl = workloads.named("mha_noncausal", seed=seed("mha_noncausal"))
    fq, fk, fv, fsc = workloads.make_qkv_fp8(fwl)
    dfq, dfk, dfv = fq.to(dev), fk.to(dev), fv.to(dev)
    fcq = torch.tensor(fwl.cu_q, dtype=torch.int32, device=dev)
    fck = torch.tensor(fwl.cu_k, dtype=torch.int32, device=dev)
    fout = torch.empty_like(dfq)
    flse = torch.empty(fwl.total_q, fwl.H, dtype=torch.float32, device=dev)

    def fstep():
        binding.varlen_attention_fwd_fp8(dfq, dfk, dfv, fcq, fck, fwl.batch, fwl.H, fwl.H_kv,
                                         fwl.max_seqlen_q, fwl.max_seqlen_k, fwl.D, fwl.causal,
                                         fwl.window, fsc["q_scale"], fsc["k_scale"], fsc["v_scale"],
                                         fsc["o_scale"], out=fout, lse=flse)

    _, _, f_max = timed(fstep, "fp8")
    fflops = accounting.attention_flops(fwl)
    f_value = sum_over_ranks(fflops * args.steps, world) / f_max / 1e12
    # E4M3 dense tensor peak: the measured bf16 peak times the nominal fp8 / bf16 ratio (4.5 / 2.25)
    fp8_peak = peak * 2.0
    del dfq, dfk, dfv, fout, flse, fq, fk, fv

    # ---- backward pass (dq, dk, dv from the forward's out and lse) on two workloads
    backward = {}
    for name in BACKWARD_CONFIGS:
        bwl = workloads.named(name, seed=seed(name))
        _, bd = _inputs_on(bwl, dev)
        bq, bk, bv, bcq, bck = bd
        gen = torch.Generator().manual_seed(workloads.WORKLOAD_SEEDS[name] + 7 + rank)
        ddo = torch.randn(bwl.total_q, bwl.H, bwl.D, generator=gen).to(torch.bfloat16).to(dev)
        bout = torch.empty_like(bq)
        blse = torch.empty(bwl.total_q, bwl.H, dtype=torch.float32, device=dev)
        _fwd_call(bwl, bd, bout, blse)()
        gq, gk, gv = torch.empty_like(bq), torch.empty_like(bk), torch.empty_like(bv)

        def bstep():
            binding.varlen_attention_bwd(ddo, bq, bk, bv, bout, blse, bcq, bck, bwl.batch, bwl.H,
                                         bwl.H_kv, bwl.max_seqlen_q, bwl.max_seqlen_k, bwl.D,
                                         bwl.causal, bwl.window, dq=gq, dk=gk, dv=gv)

        _, _, b_max = timed(bstep, "bwd:" + name)
        bflops = accounting.backward_flops(bwl)
        b_value = sum_over_ranks(bflops * args.steps, world) / b_max / 1e12
        backward[name] = {
            "workload": name, "entry": "varlen_attention_bwd", "value": b_value, "unit": "TFLOP/s",
            "ms_per_step": b_max / args.steps * 1e3, "flops_per_step_per_gpu": bflops,
            "roofline": _tensor_roofline(b_value / world, peak, pk,
                                         kernel="bwd_dq_kernel + bwd_dkdv_kernel (same call)"),
            "gpu_launches": launches["bwd:" + name]}
        del bd, bq, bk, bv, ddo, bout, blse, gq, gk, gv

    # ---- end to end on the headline workload through the host-buffer entry point
    # (pinned memory; copies in and out inside the timed region)
    del d
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    cqh = torch.tensor(wl.cu_q, dtype=torch.int32)
    ckh = torch.tensor(wl.cu_k, dtype=torch.int32)
    outh = torch.empty_like(q).pin_memory()
    lseh = torch.empty(wl.total_q, wl.H, dtype=torch.float32).pin_memory()

    def estep():
        binding.varlen_attention_fwd_host(qh, kh, vh, cqh, ckh, wl.batch, wl.H, wl.H_kv,
                                          wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal,
                                          wl.window, outh, lseh)

    _, _, e_max = timed(estep, "e2e")
    clk.__exit__(None, None, None)
    flops = head["flops_per_step_per_gpu"]
    e_value = sum_over_ranks(flops * args.steps, world) / e_max / 1e12
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
    config = {k2: v2 for k2, v2 in head.items()
              if k2 not in ("value", "unit", "ms_per_step", "roofline", "gpu_launches")}
    config.update({"parallelism": f"dp{world}",
                   "l2": "inputs larger than L2, and a 256 MiB buffer written before every step, "
                         "outside the step events"})
    return {
        "metric": METRIC, "value": head["value"], "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config,
        "roofline": head["roofline"],
        "prefill_configs": prefill_configs,
        "decode": {"workload": "decode", **dwl.describe(), "value": d_value, "unit": "GB/s",
                   "ms_per_step": d_max / args.steps * 1e3, "bytes_per_step": dbytes,
                   "roofline": {"bound": "hbm", "achieved": d_value / world,
                                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": d_frac,
                                "peak_kind": f"{peak_kind} copy",
                                "kernel": "decode_stream_kernel<128> (+ combine and counter reset, same call)",
                                "traffic": recorded_traffic("decode_stream_kernel", "decode")},
                   "gpu_launches": launches["decode"]},
        "chunked_prefill": chunked,
        "fp8": {"workload": "mha_noncausal", "entry": "varlen_attention_fwd_fp8", "dtype": "e4m3",
                "scales": fsc, "value": f_value, "unit": "TFLOP/s",
                "ms_per_step": f_max / args.steps * 1e3, "flops_per_step_per_gpu": fflops,
                "roofline": {"bound": "tensor", "achieved": f_value / world, "peak": fp8_peak,
                             "unit": "TFLOP/s", "frac": f_value / world / fp8_peak,
                             "peak_kind": f"{peak_kind} bf16 burst x 2 (nominal e4m3 / bf16 ratio)",
                             "kernel": "prefill_fwd_kernel<128, E4M3> (+ schedule build, same call)"},
                "gpu_launches": launches["fp8"]},
        "backward": backward,
        "e2e": {"value": e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "entry": "varlen_attention_fwd_host",
                "workload": args.workload, "gpu_launches": launches["e2e"]},
        "gpu_launches": launches[args.workload],
        "clocks": clocks,
        "cpu_baseline": cpu,
        "step_ms": [round(x, 4) for x in step_ms],
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="sliding_window", choices=list(workloads.WORKLOAD_SEEDS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--no-clock-sampler", action="store_true")
    ap.add_argument("--scale", type=float, default=1.0,
                    help="shrink every sequence length (profiling captures of a small case)")
    ap.add_argument("--first-seqs", type=int, default=0,
                    help="profiling: keep only the first N sequences of the workload")
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
