"""Algorithmic work of a workload: what the benchmark divides by.

FLOPs count only the (query, key) pairs a query can see under the causal /
sliding-window band, 2 flops per multiply-add in each of QK^T and PV
(boostr flash.rs, FlashAttentionOps docs, "Sliding window": tiles outside
the window are skipped, so their work is not counted).  Bytes count K and V
once plus Q, O and logsumexp: the traffic of a pass that streams each K/V row
from HBM exactly once.
"""
from __future__ import annotations

from .workloads import Workload


def visible_pairs(wl: Workload) -> int:
    """Number of (query, key) pairs a single head attends to, summed over sequences.

    Counts, per query row i of each sequence, the keys j in [0, L_k) with
    j <= i + delta (causal or windowed) and j >= i + delta - W + 1 (windowed),
    delta = L_k - L_q, in closed form per row range.
    """
    total = 0
    for Lq, Lk in zip(wl.lengths_q, wl.lengths_k):
        if Lq == 0 or Lk == 0:
            continue
        delta = Lk - Lq
        if not wl.causal and wl.window == 0:
            total += Lq * Lk
            continue
        for i in range(Lq):
            hi = min(Lk - 1, i + delta)
            lo = max(0, i + delta - wl.window + 1) if wl.window > 0 else 0
            if hi >= lo:
                total += hi - lo + 1
    return total


def attention_flops(wl: Workload) -> float:
    """Algorithmic FLOPs: 4 * visible pairs * D * H (QK^T and PV, 2 flops per MAC)."""
    return 4.0 * visible_pairs(wl) * wl.D * wl.H


def backward_flops(wl: Workload) -> float:
    """Algorithmic FLOPs of the backward pass: 10 * visible pairs * D * H, the five
    products S = QK^T (recomputed), dP = dO V^T, dV = P^T dO, dK = dS^T Q and
    dQ = dS K at 2 flops per multiply-add (2.5 x the forward)."""
    return 10.0 * visible_pairs(wl) * wl.D * wl.H


def decode_bytes(wl: Workload) -> int:
    """Algorithmic HBM bytes of one pass: K and V once, Q, O (bf16) and LSE (f32)."""
    kv = 2 * wl.total_k * wl.H_kv * wl.D * 2
    qo = 2 * wl.total_q * wl.H * wl.D * 2
    lse = wl.total_q * wl.H * 4
    cu = 2 * (wl.batch + 1) * 4
    return kv + qo + lse + cu
