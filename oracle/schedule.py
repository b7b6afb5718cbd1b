"""CPU statement of the tile work list (test infrastructure only).

The GPU path splits every sequence's queries into blocks of ``BLOCK_M`` rows
(one work item each) and walks keys in tiles of ``BLOCK_N``.  For each query
block it needs the half-open range of key tiles [kt_lo, kt_hi) that holds
every key visible to any row of the block; the tiles outside it are skipped (boostr flash.rs,
FlashAttentionOps docs, "Sliding window": whole K/V tiles outside the window
are skipped).  The list is ordered longest first: by descending tile count,
ties by ascending (sequence, query block).  This module computes that list
from host cu_seqlens with plain Python so that the device-built list can be
compared with it entry by entry.  The bf16 path lists apart, after all
others, the tiles holding a row that sees at most 256 keys (a second kernel
variant serves them with a finer product of the softmax weights).

Visibility follows the readings used by the fp64 oracle: bottom-right causal
alignment (delta = L_k - L_q), a window of exactly W keys ending at the
diagonal, and W > 0 bounding keys above by the diagonal.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

BLOCK_M = 256
BLOCK_N = 128
RESIDUAL_MAX_KEYS = 256  # a row seeing this many keys or fewer is a "few-key" row


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


def tile_has_few_key_row(L_q: int, L_k: int, qt: int, causal: bool, window: int,
                         max_keys: int = RESIDUAL_MAX_KEYS, block_m: int = BLOCK_M) -> bool:
    """Does some row of query tile qt see between 1 and max_keys keys?  Rows are
    scanned one by one with the same visibility rules."""
    delta = L_k - L_q
    for i in range(qt * block_m, min(L_q, (qt + 1) * block_m)):
        hi = L_k - 1
        if causal or window > 0:
            hi = min(hi, i + delta)
        lo = max(0, i + delta - window + 1) if window > 0 else 0
        if 1 <= hi - lo + 1 <= max_keys:
            return True
    return False


def schedule(cu_q: Sequence[int], cu_k: Sequence[int], causal: bool, window: int,
             block_m: int = BLOCK_M, block_n: int = BLOCK_N,
             split_few_keys: bool = True) -> List[Tuple[int, int, int, int]]:
    """Sorted list of (b, qt, kt_lo, kt_hi) over every query tile of every sequence.

    With split_few_keys, the tiles holding a row that sees 1..RESIDUAL_MAX_KEYS
    keys come after all others (they are served by a second kernel variant);
    within each part: descending tile count, ties by ascending (b, qt)."""
    items = []
    for b in range(len(cu_q) - 1):
        L_q = cu_q[b + 1] - cu_q[b]
        L_k = cu_k[b + 1] - cu_k[b]
        n_qt = (L_q + block_m - 1) // block_m
        for qt in range(n_qt):
            lo, hi = query_tile_key_range(L_q, L_k, qt, causal, window, block_m, block_n)
            few = split_few_keys and tile_has_few_key_row(L_q, L_k, qt, causal, window,
                                                          block_m=block_m)
            items.append((few, b, qt, lo, hi))
    items.sort(key=lambda it: (it[0], -(it[4] - it[3]), it[1], it[2]))
    return [it[1:] for it in items]
