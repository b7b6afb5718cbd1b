// Device-side builder of the longest-first query-block list (one CTA).
#pragma once

#include "schedule.cuh"
#include "status.cuh"

namespace va {

constexpr int kBuildThreads = 1024;

// Exclusive scan of one value per thread; also returns the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* red, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    __syncthreads();
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    int before = 0;
    total = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        if (w < warp) before += red[w];
        total += red[w];
    }
    __syncthreads();
    return before + incl - v;
}

// Orders of a list: a 32-bit major key (smaller first), ties by ascending
// (sequence, tile), i.e. by enumeration order, so every order is strict.
// The forward's: descending key-tile count.
struct CostOrder {
    __device__ __forceinline__ uint32_t major(const TileEntry& e) const {
        return 0xFFFFFFFFu - static_cast<uint32_t>(e.kt_hi - e.kt_lo);
    }
};
// The backward's: sequences with more 128-row tiles first (so that the items
// claimed at about the same time share their sequence's tiles in L2), within
// one by descending cost (kt_hi - kt_lo); `cu` gives the tiles' sequence lengths.
struct SeqThenCostOrder {
    const int* cu;
    __device__ __forceinline__ uint32_t major(const TileEntry& e) const {
        const uint32_t tiles = static_cast<uint32_t>((cu[e.b + 1] - cu[e.b] + kBlockM - 1) / kBlockM);
        const uint32_t cost = static_cast<uint32_t>(e.kt_hi - e.kt_lo);
        return ((0xFFFFu - min(tiles, 0xFFFFu)) << 16) | (0xFFFFu - min(cost, 0xFFFFu));
    }
};
template <class Order>
__device__ __forceinline__ bool entry_before(const TileEntry& x, const TileEntry& y, const Order& ord) {
    const uint32_t mx = ord.major(x), my = ord.major(y);
    if (mx != my) return mx < my;
    if (x.b != y.b) return x.b < y.b;
    return x.qt < y.qt;
}

// One pass of a bottom-up merge sort over `total` entries: the sorted runs
// [2 p w, 2 p w + w) and [2 p w + w, 2 p w + 2 w) of `src` are merged into
// the same range of `dst`.  The output is cut into one contiguous segment per
// thread; each thread finds, by binary search along the merge path, how many
// entries of the first run precede its segment, then merges sequentially.
template <class Order>
__device__ void merge_pass(const TileEntry* __restrict__ src, TileEntry* __restrict__ dst,
                           int total, int w, const Order& ord) {
    const int per = (total + blockDim.x - 1) / blockDim.x;
    int k = threadIdx.x * per;
    const int k_end = min(total, k + per);
    while (k < k_end) {
        const int base = static_cast<int>((static_cast<long long>(k) / (2ll * w)) * (2ll * w));
        const int a0 = base, na = max(0, min(w, total - base));
        const int b0 = base + na, nb = max(0, min(w, total - b0));
        const int pair_end = b0 + nb;
        const int kk = k - base;  // outputs of this pair before k
        // i = entries of run A among the first kk outputs
        int lo = max(0, kk - nb), hi = min(kk, na);
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (entry_before(src[a0 + mid], src[b0 + kk - 1 - mid], ord)) lo = mid + 1;
            else hi = mid;
        }
        int i = lo, j = kk - lo;
        const int stop = min(k_end, pair_end);
        for (; k < stop; ++k) {
            const bool take_a = i < na && (j >= nb || entry_before(src[a0 + i], src[b0 + j], ord));
            dst[k] = take_a ? src[a0 + i++] : src[b0 + j++];
        }
    }
}

// Sort `count` entries starting at `base` (in scratch, enumeration order) into
// out[base .. base + count) in the list's order.  Runs of key_slots entries
// are sorted in shared memory (bitonic, on unique 64-bit keys); longer ranges
// are then merged in global memory, ping-ponging between out and scratch, so
// the result always lands in out.  Whole block; ends with a barrier.
template <class Order>
__device__ void sort_range(TileEntry* __restrict__ scratch, TileEntry* __restrict__ out, int base,
                           int total, int key_slots, unsigned long long* keys, const Order& ord) {
    const int tid = threadIdx.x;
    scratch += base;
    out += base;
    if (total <= static_cast<int>(blockDim.x)) {
        // one entry per thread: its rank among the unique keys is its place
        // (one barrier instead of a bitonic network's log^2 steps)
        unsigned long long mine = 0;
        if (tid < total) {
            mine = (static_cast<unsigned long long>(ord.major(scratch[tid])) << 32) | static_cast<unsigned>(tid);
            keys[tid] = mine;
        }
        __syncthreads();
        if (tid < total) {
            int rank = 0;
            for (int j = 0; j < total; ++j) rank += keys[j] < mine ? 1 : 0;
            out[rank] = scratch[tid];
        }
        __syncthreads();
        return;
    }
    // number of merge passes after the run sort; the run sort writes to out
    // when that number is even and to scratch when it is odd, so the last
    // pass always lands in out
    const int R = key_slots;
    int passes = 0;
    for (long long w = R; w < total; w <<= 1) ++passes;
    TileEntry* run_dst = (passes & 1) ? scratch : out;
    for (int r0 = 0; r0 < total; r0 += R) {
        const int n = min(R, total - r0);
        int P = 1;
        while (P < n) P <<= 1;
        for (int e = tid; e < P; e += blockDim.x) {
            if (e < n) {
                keys[e] = (static_cast<unsigned long long>(ord.major(scratch[r0 + e])) << 32) |
                          static_cast<unsigned>(e);
            } else {
                keys[e] = ~0ull;
            }
        }
        __syncthreads();
        // bitonic sort, ascending; keys are unique so the order is fully determined
        for (int k = 2; k <= P; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int i = tid; i < P; i += blockDim.x) {
                    const int ixj = i ^ j;
                    if (ixj > i) {
                        const unsigned long long a = keys[i], c = keys[ixj];
                        const bool up = (i & k) == 0;
                        if ((a > c) == up) {
                            keys[i] = c;
                            keys[ixj] = a;
                        }
                    }
                }
                __syncthreads();
            }
        }
        if (run_dst == out) {
            for (int r = tid; r < n; r += blockDim.x)
                out[r0 + r] = scratch[r0 + static_cast<int>(keys[r] & 0xFFFFFFFFull)];
        } else {
            // in place: stage the run in out (free until the merges), then gather back
            for (int r = tid; r < n; r += blockDim.x) out[r0 + r] = scratch[r0 + r];
            __syncthreads();
            for (int r = tid; r < n; r += blockDim.x)
                scratch[r0 + r] = out[r0 + static_cast<int>(keys[r] & 0xFFFFFFFFull)];
        }
        __syncthreads();
    }
    TileEntry* src = run_dst;
    TileEntry* dst = run_dst == out ? scratch : out;
    for (long long w = R; w < total; w <<= 1) {
        merge_pass(src, dst, total, static_cast<int>(w), ord);
        __syncthreads();
        TileEntry* t = src;
        src = dst;
        dst = t;
    }
}

// The query blocks of one sequence that hold a row seeing 1..kResidualMaxKeys
// keys: [r0, r0 + nr).  Blocks before the first row that sees any key have
// none; from there on a block holds such a row exactly when its first row that
// sees a key does (counts never decrease with the row index), so these blocks
// are contiguous and the scan stops at the first block without one.
__device__ __forceinline__ void few_key_blocks(int Lq, int Lk, int n, bool causal, int window,
                                               int& r0, int& nr) {
    r0 = 0;
    nr = 0;
    if (Lq <= 0 || Lk <= 0) return;
    const int i0 = (causal || window > 0) ? max(0, Lq - Lk) : 0;  // first row that sees a key
    if (i0 >= Lq) return;
    int qt = i0 / kBlockQ;
    r0 = qt;
    while (qt < n && rows_see_few_keys(qt * kBlockQ, kBlockQ, Lq, Lk, causal, window)) ++qt;
    nr = qt - r0;
}

// Per-sequence offsets of its blocks in the two parts of the list, and its
// few-key block range (kept in the output buffer while the list is built).
struct SeqOffsets {
    int main_off, res_off, r0, nr;
};
static_assert(sizeof(SeqOffsets) == sizeof(TileEntry), "kept in the list's buffer");

// scratch: [capacity] enumeration-ordered entries; out: [capacity] sorted.
// Dynamic shared memory: 8 bytes per key slot (a power of two <= kSortCapacity).
// With split_residual, blocks that hold a row seeing 1..kResidualMaxKeys keys
// are listed after all others (hdr->n_main counts the others); each part is
// ordered longest first, ties by enumeration order.
// Enumeration: one thread per sequence finds its block counts and offsets
// (two exclusive scans); then, when the per-sequence offsets fit the output
// buffer (batch <= capacity), one thread per list entry finds its sequence by
// a binary search over them, so long sequences do not serialise on one thread.
__global__ void __launch_bounds__(kBuildThreads, 1)
build_schedule_kernel(const int* __restrict__ cu_q, const int* __restrict__ cu_k,
                      const int* __restrict__ seqused_k, int batch,
                      int causal, int window, int split_residual, int capacity, int key_slots,
                      TileEntry* __restrict__ scratch, TileEntry* __restrict__ out,
                      SchedHeader* __restrict__ hdr) {
    extern __shared__ unsigned long long keys[];
    __shared__ int red[32];
    const int tid = threadIdx.x;
    const bool cz = causal != 0;
    // the attention kernels that read this list may start their set-up now;
    // they wait for this grid's completion before their first read of the list
    grid_launch_dependents();

    const bool by_entry = batch <= capacity;
    SeqOffsets* offs = reinterpret_cast<SeqOffsets*>(out);
    int carry = 0, carry_res = 0;
    for (int base = 0; base < batch; base += blockDim.x) {
        const int b = base + tid;
        int n = 0, r0 = 0, nr = 0;
        if (b < batch) {
            const int Lq = cu_q[b + 1] - cu_q[b];
            n = (Lq + kBlockQ - 1) / kBlockQ;
            if (split_residual) few_key_blocks(Lq, seq_key_count(cu_k, seqused_k, b), n, cz, window, r0, nr);
        }
        int chunk_main, chunk_res;
        const int first = carry + block_exclusive_scan(n - nr, red, chunk_main);
        const int first_res = carry_res + block_exclusive_scan(nr, red, chunk_res);
        if (by_entry && b < batch) offs[b] = SeqOffsets{first, first_res, r0, nr};
        carry += chunk_main;
        carry_res += chunk_res;
    }
    const int n_main = carry, total = carry + carry_res;
    if (total > capacity) {
        if (tid == 0) {
            hdr->n_tiles = 0;
            hdr->next_item = 0;
            hdr->n_main = 0;
            hdr->next_item_res = 0;
            atomicOr(&g_va_status, kStatusScheduleOverflow);
        }
        return;
    }
    __syncthreads();

    if (by_entry) {
        for (int d = tid; d < total; d += blockDim.x) {
            const bool res = d >= n_main;
            const int key = res ? d - n_main : d;
            // the last sequence whose part starts at or before `key` (sequences
            // with no block in this part share the next one's offset and come
            // before it)
            int lo = 0, hi = batch - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                const int off = res ? offs[mid].res_off : offs[mid].main_off;
                if (off <= key) lo = mid;
                else hi = mid - 1;
            }
            const SeqOffsets so = offs[lo];
            const int j = key - (res ? so.res_off : so.main_off);
            const int qt = res ? so.r0 + j : (j < so.r0 ? j : j + so.nr);
            const int Lq = cu_q[lo + 1] - cu_q[lo];
            const int Lk = seq_key_count(cu_k, seqused_k, lo);
            int klo, khi;
            rows_key_range(qt * kBlockQ, kBlockQ, Lq, Lk, cz, window, klo, khi);
            scratch[d] = TileEntry{lo, qt, klo, khi};
        }
    } else {
        // more sequences than list entries (many are empty): one thread per
        // sequence writes its blocks
        carry = 0;
        carry_res = 0;
        for (int base = 0; base < batch; base += blockDim.x) {
            const int b = base + tid;
            int n = 0, r0 = 0, nr = 0, Lq = 0, Lk = 0;
            if (b < batch) {
                Lq = cu_q[b + 1] - cu_q[b];
                Lk = seq_key_count(cu_k, seqused_k, b);
                n = (Lq + kBlockQ - 1) / kBlockQ;
                if (split_residual) few_key_blocks(Lq, Lk, n, cz, window, r0, nr);
            }
            int chunk_main, chunk_res;
            const int first = carry + block_exclusive_scan(n - nr, red, chunk_main);
            const int first_res = n_main + carry_res + block_exclusive_scan(nr, red, chunk_res);
            for (int qt = 0; qt < n; ++qt) {
                int klo, khi;
                rows_key_range(qt * kBlockQ, kBlockQ, Lq, Lk, cz, window, klo, khi);
                const bool res = qt >= r0 && qt < r0 + nr;
                scratch[res ? first_res + (qt - r0) : first + (qt < r0 ? qt : qt - nr)] =
                    TileEntry{b, qt, klo, khi};
            }
            carry += chunk_main;
            carry_res += chunk_res;
        }
    }
    __syncthreads();
    sort_range(scratch, out, 0, n_main, key_slots, keys, CostOrder{});
    sort_range(scratch, out, n_main, total - n_main, key_slots, keys, CostOrder{});
    if (tid == 0) {
        hdr->n_tiles = total;
        hdr->next_item = 0;
        hdr->n_main = n_main;
        hdr->next_item_res = 0;
    }
}

// Work lists of the backward pass, one entry per 128-row tile of a sequence,
// sequences with more tiles first, within one heaviest first (ties by
// (sequence, tile)):
//   mode 0 (dQ): query tile qt, {b, qt, kt_lo, kt_hi} = its visible key tiles
//   mode 1 (dK/dV): key tile kt, {b, kt, 0, n_qt} = the number of 128-row
//                   query tiles holding a row that sees one of its keys
// Every tile of every sequence is listed (tiles with no visible pair too: their
// gradient rows are written as zeros).  hdr->n_tiles = the list's length,
// hdr->next_item = 0.  Needs batch <= capacity (the per-sequence offsets are
// kept in `out` while the list is built).
__global__ void __launch_bounds__(kBuildThreads, 1)
build_bwd_list_kernel(const int* __restrict__ cu_q, const int* __restrict__ cu_k, int batch, int causal,
                      int window, int mode, int capacity, int key_slots, TileEntry* __restrict__ scratch,
                      TileEntry* __restrict__ out, SchedHeader* __restrict__ hdr) {
    extern __shared__ unsigned long long keys[];
    __shared__ int red[32];
    const int tid = threadIdx.x;
    const bool cz = causal != 0;
    if (batch > capacity) {  // (the offsets below would not fit)
        if (tid == 0) {
            hdr->n_tiles = 0;
            hdr->next_item = 0;
            hdr->n_main = 0;
            hdr->next_item_res = 0;
            atomicOr(&g_va_status, kStatusScheduleOverflow);
        }
        return;
    }
    int* offs = reinterpret_cast<int*>(out);  // [batch]: first entry of each sequence
    int carry = 0;
    for (int base = 0; base < batch; base += blockDim.x) {
        const int b = base + tid;
        int n = 0;
        if (b < batch) {
            const int L = mode == 0 ? cu_q[b + 1] - cu_q[b] : cu_k[b + 1] - cu_k[b];
            n = (max(L, 0) + kBlockM - 1) / kBlockM;
        }
        int chunk;
        const int first = carry + block_exclusive_scan(n, red, chunk);
        if (b < batch) offs[b] = first;
        carry += chunk;
    }
    const int total = carry;
    if (total > capacity) {
        if (tid == 0) {
            hdr->n_tiles = 0;
            hdr->next_item = 0;
            hdr->n_main = 0;
            hdr->next_item_res = 0;
            atomicOr(&g_va_status, kStatusScheduleOverflow);
        }
        return;
    }
    __syncthreads();
    for (int d = tid; d < total; d += blockDim.x) {
        int lo = 0, hi = batch - 1;  // the last sequence whose tiles start at or before d
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offs[mid] <= d) lo = mid;
            else hi = mid - 1;
        }
        const int t = d - offs[lo];
        const int L_q = cu_q[lo + 1] - cu_q[lo], L_k = cu_k[lo + 1] - cu_k[lo];
        TileEntry e;
        if (mode == 0) {
            int klo, khi;
            rows_key_range(t * kBlockM, kBlockM, L_q, L_k, cz, window, klo, khi);
            e = TileEntry{lo, t, klo, khi};
        } else {
            int r0, r1;
            key_tile_rows(t, L_q, L_k, cz, window, r0, r1);
            e = TileEntry{lo, t, 0, r1 >= r0 ? r1 / kBlockM - r0 / kBlockM + 1 : 0};
        }
        scratch[d] = e;
    }
    __syncthreads();
    sort_range(scratch, out, 0, total, key_slots, keys, SeqThenCostOrder{mode == 0 ? cu_q : cu_k});
    if (tid == 0) {
        hdr->n_tiles = total;
        hdr->next_item = 0;
        hdr->n_main = total;
        hdr->next_item_res = 0;
    }
}

}  // namespace va
