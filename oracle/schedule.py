"""CPU statement of the tile work list (test infrastructure only).

The GPU path splits every sequence's queries into blocks of ``BLOCK_M`` rows
(one work item each) and walks keys in tiles of ``BLOCK_N``.  For each query
block it needs the half-open range of key tiles [kt_lo, kt_hi) that holds
every key visible to any row of the block; the tiles outside it are skipped (boostr flash.rs,
FlashAttentionOps docs, "Sliding window": whole K/V tiles outside the window
are skipped).  The list is ordered longest first: by descending tile count,
ties by ascending (sequence, query block).  This module computes that list
from host cu_seqlens with plain Python so that the device-built list can be
compared with it entry by entry.

Visibility follows the readings used by the fp64 oracle: bottom-right causal
alignment (delta = L_k - L_q), a window of exactly W keys ending at the
diagonal, and W > 0 bounding keys above by the diagonal.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

BLOCK_M = 256
BLOCK_N = 128


def query_tile_key_range(L_q: int, L_k: int, qt: int, causal: bool, window: int,
                         block_m: int = BLOCK_M, block_n: int = BLOCK_N) -> Tuple[int, int]:
    """[kt_lo, kt_hi) for query tile qt; (0, 0) when no row of it sees a key."""
    delta = L_k - L_q
    first = qt * block_m
    last = min(L_q, first + block_m) - 1
    lo_keys, hi_keys = None, None
    # rows are scanned one by one: the union of their visible key intervals
    for i in range(first, last + 1):
        hi = L_k - 1
        if causal or window > 0:
            hi = min(hi, i + delta)
        lo = 0
        if window > 0:
            lo = max(0, i + delta - window + 1)
        if lo > hi:
            continue
        lo_keys = lo if lo_keys is None else min(lo_keys, lo)
        hi_keys = hi if hi_keys is None else max(hi_keys, hi)
    if lo_keys is None:
        return 0, 0
    return lo_keys // block_n, hi_keys // block_n + 1


def schedule(cu_q: Sequence[int], cu_k: Sequence[int], causal: bool, window: int,
             block_m: int = BLOCK_M, block_n: int = BLOCK_N) -> List[Tuple[int, int, int, int]]:
    """Sorted list of (b, qt, kt_lo, kt_hi) over every query tile of every sequence."""
    items = []
    for b in range(len(cu_q) - 1):
        L_q = cu_q[b + 1] - cu_q[b]
        L_k = cu_k[b + 1] - cu_k[b]
        n_qt = (L_q + block_m - 1) // block_m
        for qt in range(n_qt):
            lo, hi = query_tile_key_range(L_q, L_k, qt, causal, window, block_m, block_n)
            items.append((b, qt, lo, hi))
    items.sort(key=lambda it: (-(it[3] - it[2]), it[0], it[1]))
    return items
