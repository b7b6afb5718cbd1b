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

// scratch: [capacity] enumeration-ordered entries; out: [capacity] sorted.
// Dynamic shared memory: 8 bytes per key slot (a power of two <= kSortCapacity).
__global__ void __launch_bounds__(kBuildThreads, 1)
build_schedule_kernel(const int* __restrict__ cu_q, const int* __restrict__ cu_k,
                      const int* __restrict__ seqused_k, int batch,
                      int causal, int window, int capacity, int key_slots,
                      TileEntry* __restrict__ scratch, TileEntry* __restrict__ out,
                      SchedHeader* __restrict__ hdr) {
    extern __shared__ unsigned long long keys[];
    __shared__ int red[32];
    const int tid = threadIdx.x;
    // the attention kernel that reads this list may start its set-up now; it
    // waits for this grid's completion before its first read of the list
    grid_launch_dependents();

    int local = 0;
    for (int b = tid; b < batch; b += blockDim.x) {
        const int Lq = cu_q[b + 1] - cu_q[b];
        local += (Lq + kBlockQ - 1) / kBlockQ;
    }
    const int total = block_sum(local, red);
    if (total > capacity) {
        if (tid == 0) {
            hdr->n_tiles = 0;
            hdr->next_item = 0;
            atomicOr(&g_va_status, kStatusScheduleOverflow);
        }
        return;
    }
    const bool sort_in_smem = total <= key_slots;

    int carry = 0;
    for (int base = 0; base < batch; base += blockDim.x) {
        const int b = base + tid;
        int n = 0, Lq = 0, Lk = 0;
        if (b < batch) {
            Lq = cu_q[b + 1] - cu_q[b];
            Lk = seq_key_count(cu_k, seqused_k, b);
            n = (Lq + kBlockQ - 1) / kBlockQ;
        }
        int chunk_total;
        const int first = carry + block_exclusive_scan(n, red, chunk_total);
        for (int qt = 0; qt < n; ++qt) {
            int lo, hi;
            rows_key_range(qt * kBlockQ, kBlockQ, Lq, Lk, causal != 0, window, lo, hi);
            const int e = first + qt;
            scratch[e] = TileEntry{b, qt, lo, hi};
            if (sort_in_smem) {
                const unsigned inv_cost = 0xFFFFFFFFu - static_cast<unsigned>(hi - lo);
                keys[e] = (static_cast<unsigned long long>(inv_cost) << 32) | static_cast<unsigned>(e);
            }
        }
        carry += chunk_total;
    }
    __syncthreads();

    if (!sort_in_smem) {
        // beyond the shared-memory sort capacity: enumeration order
        for (int e = tid; e < total; e += blockDim.x) out[e] = scratch[e];
        if (tid == 0) {
            hdr->n_tiles = total;
            hdr->next_item = 0;
        }
        return;
    }
    int P = 1;
    while (P < total) P <<= 1;
    for (int e = total + tid; e < P; e += blockDim.x) keys[e] = ~0ull;
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
    for (int r = tid; r < total; r += blockDim.x) {
        out[r] = scratch[static_cast<int>(keys[r] & 0xFFFFFFFFull)];
    }
    if (tid == 0) {
        hdr->n_tiles = total;
        hdr->next_item = 0;
    }
}

}  // namespace va
