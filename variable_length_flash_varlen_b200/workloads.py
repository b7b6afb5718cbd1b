"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no attention arithmetic: it draws sequence lengths, forms
the cumulative-length index the packed layout is addressed by, and draws
bf16 Q/K/V ~ N(0, 1).  Both the CUDA path and the fp64 oracle take its
outputs as inputs.

Packed layout (boostr 0.2.0 varlen_attention.rs, VarLenAttentionOps docs,
"Layout contract" and "Cumulative sequence lengths"): q is
[total_q, H, D], k and v are [total_k, H_kv, D], and cu_seqlens is the int32
exclusive prefix sum of the lengths with a leading 0, e.g. lengths
[512, 300, 128] give [0, 512, 812, 940].

Named workloads (all bf16, Q/K/V ~ N(0, 1), softmax scale 1/sqrt(D)):
  worked_example   lengths [512, 300, 128] for q and k, H=4, H_kv=2, D=64, causal
  mha_noncausal    16 sequences, q = k lengths uniform-int in [64, 2048],
                   H = H_kv = 16, D=128
  gqa_causal       lengths round(exp(U[ln 128, ln 8192])) drawn while the sum
                   is below 65536, the last one then set so the sum is exactly
                   65536; H=32, H_kv=8, D=128, causal
  sliding_window   4 sequences of 32768, window 4096, causal, H=32, H_kv=8, D=128
  decode           128 sequences, q length 1, k lengths uniform-int in
                   [1024, 32768], non-causal, H=32, H_kv=8, D=128
  chunked_prefill  32 sequences, each a new chunk of q length uniform-int in
                   [128, 1024] appended to a cached prefix of uniform-int
                   [0, 8192] keys (k length = prefix + chunk), causal with the
                   diagonal at the end of the keys, H=32, H_kv=8, D=128
Lengths come from random.Random(seed); Q, K, V (in that order) from a torch
CPU generator seeded with the same seed, drawn in fixed-size chunks.

FP8 inputs (``make_qkv_fp8``): the same N(0, 1) draws divided by a per-tensor
scale of 2^-6 and rounded to E4M3 (torch's float8_e4m3fn conversion), so the
codes span about +-350 of E4M3's +-448 and each element's value is code *
2^-6; the output scale is 2^-5 (output code = O / o_scale), which keeps
|O| / o_scale <= 448 for any output (|O| <= max |v| < 14 here).
"""
from __future__ import annotations

import math
import random
from dataclasses import dataclass, field
from typing import List, Optional

import torch

CHUNK = 1 << 24  # elements per randn draw (bounds the fp32 temporary)

WORKLOAD_SEEDS = {
    "worked_example": 1001,
    "mha_noncausal": 1002,
    "gqa_causal": 1003,
    "sliding_window": 1004,
    "decode": 1005,
    "chunked_prefill": 1006,
}


@dataclass
class Workload:
    name: str
    lengths_q: List[int]
    lengths_k: List[int]
    H: int
    H_kv: int
    D: int
    causal: bool
    window: int
    seed: int
    cu_q: List[int] = field(init=False)
    cu_k: List[int] = field(init=False)

    def __post_init__(self):
        if len(self.lengths_q) != len(self.lengths_k):
            raise ValueError("lengths_q and lengths_k must have one entry per sequence")
        self.cu_q = cu_seqlens(self.lengths_q)
        self.cu_k = cu_seqlens(self.lengths_k)

    @property
    def batch(self) -> int:
        return len(self.lengths_q)

    @property
    def total_q(self) -> int:
        return self.cu_q[-1]

    @property
    def total_k(self) -> int:
        return self.cu_k[-1]

    @property
    def max_seqlen_q(self) -> int:
        return max(self.lengths_q) if self.lengths_q else 0

    @property
    def max_seqlen_k(self) -> int:
        return max(self.lengths_k) if self.lengths_k else 0

    def describe(self) -> dict:
        return {"workload": self.name, "batch": self.batch, "total_q": self.total_q,
                "total_k": self.total_k, "H": self.H, "H_kv": self.H_kv, "D": self.D,
                "causal": self.causal, "window": self.window, "seed": self.seed}


def cu_seqlens(lengths: List[int]) -> List[int]:
    """Exclusive prefix sum with a leading zero (the packed-layout index)."""
    out = [0]
    for n in lengths:
        if n < 0:
            raise ValueError("sequence lengths must be non-negative")
        out.append(out[-1] + int(n))
    if out[-1] >= 2 ** 31:
        raise ValueError("total tokens must fit in int32")
    return out


def _randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    n = 1
    for s in shape:
        n *= s
    flat = torch.empty(n, dtype=torch.bfloat16)
    for start in range(0, n, CHUNK):
        stop = min(n, start + CHUNK)
        flat[start:stop] = torch.randn(stop - start, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    return flat.view(*shape)


FP8_INPUT_SCALE = 2.0 ** -6   # q_scale = k_scale = v_scale: dequantized value = code * scale
FP8_OUTPUT_SCALE = 2.0 ** -5  # o_scale: output code = E4M3(O / o_scale)


def _randn_e4m3(shape, gen: torch.Generator, scale: float) -> torch.Tensor:
    """N(0, 1) / scale rounded to E4M3, as uint8 bit patterns."""
    n = 1
    for s in shape:
        n *= s
    flat = torch.empty(n, dtype=torch.uint8)
    for start in range(0, n, CHUNK):
        stop = min(n, start + CHUNK)
        x = torch.randn(stop - start, generator=gen, dtype=torch.float32) / scale
        flat[start:stop] = x.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return flat.view(*shape)


def make_qkv_fp8(wl: Workload):
    """E4M3 q [total_q, H, D], k and v [total_k, H_kv, D] (uint8 bit patterns) and the
    four scales of the FP8 forward, drawn from wl.seed."""
    gen = torch.Generator(device="cpu").manual_seed(wl.seed)
    q = _randn_e4m3((wl.total_q, wl.H, wl.D), gen, FP8_INPUT_SCALE)
    k = _randn_e4m3((wl.total_k, wl.H_kv, wl.D), gen, FP8_INPUT_SCALE)
    v = _randn_e4m3((wl.total_k, wl.H_kv, wl.D), gen, FP8_INPUT_SCALE)
    scales = {"q_scale": FP8_INPUT_SCALE, "k_scale": FP8_INPUT_SCALE,
              "v_scale": FP8_INPUT_SCALE, "o_scale": FP8_OUTPUT_SCALE}
    return q, k, v, scales


def make_qkv(wl: Workload, device: str = "cpu"):
    """bf16 q [total_q, H, D], k and v [total_k, H_kv, D] drawn from wl.seed."""
    gen = torch.Generator(device="cpu").manual_seed(wl.seed)
    q = _randn_bf16((wl.total_q, wl.H, wl.D), gen)
    k = _randn_bf16((wl.total_k, wl.H_kv, wl.D), gen)
    v = _randn_bf16((wl.total_k, wl.H_kv, wl.D), gen)
    if device != "cpu":
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


def _uniform_lengths(rng: random.Random, n: int, lo: int, hi: int) -> List[int]:
    return [rng.randint(lo, hi) for _ in range(n)]


def _log_uniform_until(rng: random.Random, lo: int, hi: int, total: int) -> List[int]:
    out: List[int] = []
    while sum(out) < total:
        out.append(int(round(math.exp(rng.uniform(math.log(lo), math.log(hi))))))
    out[-1] = total - sum(out[:-1])
    return out


def named(name: str, seed: Optional[int] = None, scale: float = 1.0) -> Workload:
    """A named workload; ``scale`` < 1 shrinks every length (parity-test sizes)."""
    s = WORKLOAD_SEEDS[name] if seed is None else seed
    rng = random.Random(s)

    def shrink(xs):
        return [max(1, int(round(x * scale))) for x in xs] if scale != 1.0 else xs

    if name == "worked_example":
        L = shrink([512, 300, 128])
        return Workload(name, L, L, 4, 2, 64, True, 0, s)
    if name == "mha_noncausal":
        L = shrink(_uniform_lengths(rng, 16, 64, 2048))
        return Workload(name, L, L, 16, 16, 128, False, 0, s)
    if name == "gqa_causal":
        L = shrink(_log_uniform_until(rng, 128, 8192, 65536))
        return Workload(name, L, L, 32, 8, 128, True, 0, s)
    if name == "sliding_window":
        L = shrink([32768] * 4)
        W = max(1, int(round(4096 * scale)))
        return Workload(name, L, L, 32, 8, 128, True, W, s)
    if name == "decode":
        Lk = shrink(_uniform_lengths(rng, 128, 1024, 32768))
        return Workload(name, [1] * 128, Lk, 32, 8, 128, False, 0, s)
    if name == "chunked_prefill":
        Lq = _uniform_lengths(rng, 32, 128, 1024)
        prefix = _uniform_lengths(rng, 32, 0, 8192)
        Lq_s, pre_s = shrink(Lq), [int(round(x * scale)) for x in prefix]
        return Workload(name, Lq_s, [a + b for a, b in zip(Lq_s, pre_s)], 32, 8, 128, True, 0, s)
    raise KeyError(name)


def custom(lengths_q: List[int], lengths_k: List[int], H: int, H_kv: int, D: int,
           causal: bool, window: int, seed: int, name: str = "custom") -> Workload:
    return Workload(name, list(lengths_q), list(lengths_k), H, H_kv, D, causal, window, seed)
