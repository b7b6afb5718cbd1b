// Device-side builder of the longest-first query-block list (one CTA).
#pragma once

#include "schedule.cuh"
#include "status.cuh"

namespace va {

constexpr int kBuildThreads = 1024;

__device__ __forceinline__ int block_sum(int v, int* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    __syncthreads();
    return t;
}

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

// Strict order of the list: descending key-tile count, ties by ascending
// (sequence, query block), i.e. by enumeration order.
__device__ __forceinline__ bool entry_before(const TileEntry& x, const TileEntry& y) {
    const int cx = x.kt_hi - x.kt_lo, cy = y.kt_hi - y.kt_lo;
    if (cx != cy) return cx > cy;
    if (x.b != y.b) return x.b < y.b;
    return x.qt < y.qt;
}

// One pass of a bottom-up merge sort over `total` entries: the sorted runs
// [2 p w, 2 p w + w) and [2 p w + w, 2 p w + 2 w) of `src` are merged into
// the same range of `dst`.  The output is cut into one contiguous segment per
// thread; each thread finds, by binary search along the merge path, how many
// entries of the first run precede its segment, then merges sequentially.
__device__ void merge_pass(const TileEntry* __restrict__ src, TileEntry* __restrict__ dst,
                           int total, int w) {
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
            if (entry_before(src[a0 + mid], src[b0 + kk - 1 - mid])) lo = mid + 1;
            else hi = mid;
        }
        int i = lo, j = kk - lo;
        const int stop = min(k_end, pair_end);
        for (; k < stop; ++k) {
            const bool take_a = i < na && (j >= nb || entry_before(src[a0 + i], src[b0 + j]));
            dst[k] = take_a ? src[a0 + i++] : src[b0 + j++];
        }
    }
}

// Sort `count` entries starting at `base` (in scratch, enumeration order) into
// out[base .. base + count) in the list's order.  Runs of key_slots entries
// are sorted in shared memory (bitonic, on unique 64-bit keys); longer ranges
// are then merged in global memory, ping-ponging between out and scratch, so
// the result always lands in out.  Whole block; ends with a barrier.
__device__ void sort_range(TileEntry* __restrict__ scratch, TileEntry* __restrict__ out, int base,
                           int total, int key_slots, unsigned long long* keys) {
    const int tid = threadIdx.x;
    scratch += base;
    out += base;
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
                const TileEntry te = scratch[r0 + e];
                const unsigned inv_cost = 0xFFFFFFFFu - static_cast<unsigned>(te.kt_hi - te.kt_lo);
                keys[e] = (static_cast<unsigned long long>(inv_cost) << 32) | static_cast<unsigned>(e);
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
        merge_pass(src, dst, total, static_cast<int>(w));
        __syncthreads();
        TileEntry* t = src;
        src = dst;
        dst = t;
    }
}

// scratch: [capacity] enumeration-ordered entries; out: [capacity] sorted.
// Dynamic shared memory: 8 bytes per key slot (a power of two <= kSortCapacity).
// With split_residual, blocks that hold a row seeing 1..kResidualMaxKeys keys
// are listed after all others (hdr->n_main counts the others); each part is
// ordered longest first, ties by enumeration order.
__global__ void __launch_bounds__(kBuildThreads, 1)
build_schedule_kernel(const int* __restrict__ cu_q, const int* __restrict__ cu_k,
                      const int* __restrict__ seqused_k, int batch,
                      int causal, int window, int split_residual, int capacity, int key_slots,
                      TileEntry* __restrict__ scratch, TileEntry* __restrict__ out,
                      SchedHeader* __restrict__ hdr) {
    extern __shared__ unsigned long long keys[];
    __shared__ int red[32];
    const int tid = threadIdx.x;
    // the attention kernels that read this list may start their set-up now;
    // they wait for this grid's completion before their first read of the list
    grid_launch_dependents();

    // blocks of a sequence that need the residual product
    auto residual_blocks = [&](int Lq, int Lk, int n) {
        int r = 0;
        if (split_residual)
            for (int qt = 0; qt < n; ++qt)
                r += rows_see_few_keys(qt * kBlockQ, kBlockQ, Lq, Lk, causal != 0, window) ? 1 : 0;
        return r;
    };
    int local = 0, local_res = 0;
    for (int b = tid; b < batch; b += blockDim.x) {
        const int Lq = cu_q[b + 1] - cu_q[b];
        const int n = (Lq + kBlockQ - 1) / kBlockQ;
        local += n;
        local_res += residual_blocks(Lq, seq_key_count(cu_k, seqused_k, b), n);
    }
    const int total = block_sum(local, red);
    const int total_res = block_sum(local_res, red);
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
    const int n_main = total - total_res;

    // enumeration, partitioned: the first part at [0, n_main), the blocks that
    // need the residual product at [n_main, total), each in enumeration order
    int carry = 0, carry_res = 0;
    for (int base = 0; base < batch; base += blockDim.x) {
        const int b = base + tid;
        int n = 0, nr = 0, Lq = 0, Lk = 0;
        if (b < batch) {
            Lq = cu_q[b + 1] - cu_q[b];
            Lk = seq_key_count(cu_k, seqused_k, b);
            n = (Lq + kBlockQ - 1) / kBlockQ;
            nr = residual_blocks(Lq, Lk, n);
        }
        int chunk_main, chunk_res;
        const int first = carry + block_exclusive_scan(n - nr, red, chunk_main);
        const int first_res = n_main + carry_res + block_exclusive_scan(nr, red, chunk_res);
        int im = first, ir = first_res;
        for (int qt = 0; qt < n; ++qt) {
            int lo, hi;
            rows_key_range(qt * kBlockQ, kBlockQ, Lq, Lk, causal != 0, window, lo, hi);
            const bool res = split_residual &&
                             rows_see_few_keys(qt * kBlockQ, kBlockQ, Lq, Lk, causal != 0, window);
            scratch[res ? ir++ : im++] = TileEntry{b, qt, lo, hi};
        }
        carry += chunk_main;
        carry_res += chunk_res;
    }
    __syncthreads();
    sort_range(scratch, out, 0, n_main, key_slots, keys);
    sort_range(scratch, out, n_main, total_res, key_slots, keys);
    if (tid == 0) {
        hdr->n_tiles = total;
        hdr->next_item = 0;
        hdr->n_main = n_main;
        hdr->next_item_res = 0;
    }
}

}  // namespace va
