// Work list of query tiles, built on the device from cu_seqlens.
//
// Every sequence b's queries are cut into blocks of kBlockQ rows (one work
// item; the kernel splits it into two MMA tiles of kBlockM rows); for each
// block the key tiles (kBlockN keys) that any of its rows can see form the
// half-open range [kt_lo, kt_hi).  Key tiles outside the range are never
// loaded: the causal triangle above the diagonal and the keys older than a
// sliding window (boostr flash.rs, FlashAttentionOps docs, "Sliding window")
// cost nothing.  The list is sorted longest first (descending kt_hi - kt_lo,
// ties by ascending (b, query tile)) so a persistent grid starts with the
// heaviest tiles and finishes with the light ones.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace va {

constexpr int kBlockM = 128;   // query rows per MMA tile
constexpr int kBlockQ = 256;   // query rows per work item (two MMA tiles)
constexpr int kBlockN = 128;   // keys per tile
constexpr int kSortCapacity = 16384;  // query blocks sorted in shared memory

struct TileEntry {
    int b, qt, kt_lo, kt_hi;  // sequence, query block, key-tile range of the block
};

// Visible key interval [lo, hi] of query row i (sequence-relative) under the
// readings used throughout: delta = L_k - L_q aligns the causal diagonal to
// the bottom-right, and a window of W > 0 keeps exactly the W keys ending at
// the diagonal.  Empty when lo > hi.
__host__ __device__ __forceinline__ void row_key_interval(int i, int L_q, int L_k, bool causal,
                                                          int window, int& lo, int& hi) {
    const int diag = i + (L_k - L_q);
    hi = L_k - 1;
    if (causal || window > 0) hi = diag < hi ? diag : hi;
    lo = 0;
    if (window > 0) {
        const int w0 = diag - window + 1;
        lo = w0 > 0 ? w0 : 0;
    }
}

// Keys of sequence b: its rows cu_k[b]..cu_k[b+1]-1, or, for a key-value cache
// with a capacity stride (flash.rs FlashAttentionOps docs, "kv_seq_len": iterate
// over the first n positions while the buffer size stays the stride), only the
// first seqused_k[b] of them (clamped to that range) when seqused_k is given.
__host__ __device__ __forceinline__ int seq_key_count(const int* cu_k, const int* seqused_k, int b) {
    const int cap = cu_k[b + 1] - cu_k[b];
    if (!seqused_k) return cap;
    const int used = seqused_k[b] > 0 ? seqused_k[b] : 0;
    return used < cap ? used : cap;
}

// Query rows of a sequence that see some key of key tile kt (keys [k0,
// k_last]): [r0, r1] under bottom-right causal alignment and a window of W
// keys ending at the diagonal (empty when r1 < r0).
__host__ __device__ __forceinline__ void key_tile_rows(int kt, int L_q, int L_k, bool causal, int window,
                                                       int& r0, int& r1) {
    const int k0 = kt * kBlockN;
    const int k_last = (L_k < k0 + kBlockN ? L_k : k0 + kBlockN) - 1;
    const int delta_k = L_k - L_q;
    r0 = 0;
    r1 = L_q - 1;
    if (causal || window > 0) r0 = (k0 - delta_k > 0 ? k0 - delta_k : 0);
    if (window > 0) r1 = (r1 < k_last - delta_k + window - 1 ? r1 : k_last - delta_k + window - 1);
    if (L_q <= 0 || k0 >= L_k) r1 = r0 - 1;
}

// Key-tile range of query rows [first, first + rows) clipped to L_q.  The
// intervals of consecutive rows have non-decreasing ends and overlap or
// touch, so the union over the rows is the interval of the first non-empty
// row to the last row.  (0, 0) when no row sees a key.
__host__ __device__ __forceinline__ void rows_key_range(int first, int rows, int L_q, int L_k,
                                                        bool causal, int window, int& kt_lo,
                                                        int& kt_hi) {
    kt_lo = kt_hi = 0;
    if (L_k <= 0) return;
    const int last = min(L_q, first + rows) - 1;
    if (last < first) return;
    // first row whose interval is non-empty: diag >= 0 when the band is bounded above
    int r0 = first;
    if (causal || window > 0) {
        const int need = L_q - L_k;  // diag >= 0  <=>  i >= L_q - L_k
        if (need > r0) r0 = need;
    }
    if (r0 > last) return;
    int lo0, hi0, lo1, hi1;
    row_key_interval(r0, L_q, L_k, causal, window, lo0, hi0);
    row_key_interval(last, L_q, L_k, causal, window, lo1, hi1);
    if (hi1 < lo0) return;
    kt_lo = lo0 / kBlockN;
    kt_hi = hi1 / kBlockN + 1;
}

// A row that sees at most this many keys puts most of its softmax weight on a
// few of them, and there the bf16 rounding of P (2^-9 relative per weight) no
// longer averages out: its output can move by ~2^-9 |v|, beyond what a bf16
// result may differ from the exact one.  Query blocks holding such a row are
// listed apart and run by a kernel variant that also multiplies V by the
// residual P - bf16(P), rounded to bf16 (~2^-17 relative).
constexpr int kResidualMaxKeys = 256;

// Does some row of [first, first + rows) (clipped to L_q) see between 1 and
// kResidualMaxKeys keys?  The visible count of a row never decreases with the
// row index (the band's upper end moves with the diagonal, its width is
// fixed), so the first row that sees any key has the fewest.
__host__ __device__ __forceinline__ bool rows_see_few_keys(int first, int rows, int L_q, int L_k,
                                                           bool causal, int window) {
    int i0 = first;
    if ((causal || window > 0) && L_q - L_k > i0) i0 = L_q - L_k;
    const int end = L_q < first + rows ? L_q : first + rows;
    if (i0 >= end) return false;
    int lo, hi;
    row_key_interval(i0, L_q, L_k, causal, window, lo, hi);
    return hi >= lo && hi - lo + 1 <= kResidualMaxKeys;
}

// Workspace header written by the builder and read by the attention kernels.
// The list holds n_main blocks first, then n_tiles - n_main blocks that hold a
// row seeing few keys (each part longest first); each part has its own work
// counter, claimed by its own kernel variant.
struct SchedHeader {
    int n_tiles;        // number of valid entries in the sorted list
    int next_item;      // work counter over the first part (zeroed by the builder)
    int n_main;         // entries of the first part
    int next_item_res;  // work counter over the second part (zeroed by the builder)
};

}  // namespace va
