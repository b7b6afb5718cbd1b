// Persistent, warp-specialised packed-attention forward for sm_100a.
//
// Per CTA (192 threads, one CTA per SM):
//   warp 0      producer: TMA tile loads of Q, K, V into 128-byte-swizzled
//               shared memory (plain loads for a tile that runs past the end
//               of the packed tensor)
//   warp 1      tensor-memory owner and MMA issuer: one lane issues
//               S = Q K^T (SS form) and O += P V (P read from tensor memory)
//   warps 2-5   softmax: one query row per thread; online softmax in base 2
//               with a lazily moved reference max, P written back to tensor
//               memory as bf16, O rescaled in place, epilogue O / l and
//               logsumexp
// Tensor memory (512 columns): S/P double buffer at columns 0 and 128, O at 256.
//
// The recurrence is the tiled one of realizar 0.8.4 attention.rs, IMP-111
// (online_softmax / tiled_single_head_attention): running max, running sum
// rescaled by exp(old - new), output rescaled alongside, normalised at the end.
// Packed addressing and GQA head mapping follow boostr 0.2.0
// varlen_attention.rs, VarLenAttentionOps docs ("Layout contract", "GQA
// key/value head mapping"): kv_head = q_head / (H / H_kv), K/V read once per
// tile for the head that needs them, never repeated in memory.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"
#include "status.cuh"

namespace va {

constexpr int kPrefillThreads = 192;
constexpr int kStages = 2;             // K/V ring depth
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may grow to 2^8 before O is rescaled

struct PrefillParams {
    const int* cu_q;
    const int* cu_k;
    int batch, H, H_kv, causal, window;
    const TileEntry* tiles;
    const SchedHeader* hdr;
    int tile_capacity;  // entries the list can hold; the count read from hdr is clamped to it
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    __nv_bfloat16* out;
    float* lse;
    float scale_log2;  // log2(e) / sqrt(D)
};

template <int D>
struct PrefillSmem {
    static constexpr int kChunks = D / 64;                 // 128-byte swizzle atoms per row
    static constexpr int kChunkBytes = 128 * 128;          // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kTileBytes;
    static constexpr int kV = kK + kStages * kTileBytes;
    static constexpr int kBar = kV + kStages * kTileBytes;
    // barriers: q_full, q_empty, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2], o_done
    static constexpr int kNumBars = 2 + 4 * kStages + 5;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    // slack for 1024-byte alignment; never below 120 KB so that at most one CTA
    // (and one 512-column tensor-memory allocation) is resident per SM
    static constexpr int kAlloc = (kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024;
};

// Copy a 128-row tile whose rows may run past `T` with plain loads, writing
// the 128-byte-swizzle layout TMA would have produced; rows >= T become zero.
template <int D>
__device__ __forceinline__ void load_tile_plain(uint8_t* dst, const __nv_bfloat16* src, int row0,
                                                int T, int row_stride, int col0, int lane) {
    constexpr int kVecPerRow = D / 8;  // 16-byte vectors per row
    for (int idx = lane; idx < 128 * kVecPerRow; idx += 32) {
        const int r = idx / kVecPerRow, c = idx % kVecPerRow;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (row0 + r < T) {
            val = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(row0 + r) * row_stride +
                                                  col0 + c * 8);
        }
        const int sub = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4*>(dst + sub * PrefillSmem<D>::kChunkBytes + r * 128 +
                                  ((cc ^ (r & 7)) << 4)) = val;
    }
    fence_proxy_async_smem();
    __syncwarp();
}

template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map,
                                          const __nv_bfloat16* src, int row0, int T, int row_stride,
                                          int col0, uint64_t* full, int lane) {
    if (row0 + 128 <= T) {
        if (lane == 0) {
            mbar_arrive_expect_tx(full, PrefillSmem<D>::kTileBytes);
#pragma unroll
            for (int c = 0; c < PrefillSmem<D>::kChunks; ++c)
                tma_load_2d(dst + c * PrefillSmem<D>::kChunkBytes, map, col0 + c * 64, row0, full);
        }
        __syncwarp();
    } else {
        load_tile_plain<D>(dst, src, row0, T, row_stride, col0, lane);
        if (lane == 0) mbar_arrive(full);
        __syncwarp();
    }
}

template <int D>
__global__ void __launch_bounds__(kPrefillThreads, 1)
prefill_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
    using L = PrefillSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;
    uint64_t* k_full = bars + 2;
    uint64_t* k_empty = k_full + kStages;
    uint64_t* v_full = k_empty + kStages;
    uint64_t* v_empty = v_full + kStages;
    uint64_t* s_full = v_empty + kStages;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_done = p_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
        }
        mbar_init(o_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int n_items = min(max(p.hdr->n_tiles, 0), p.tile_capacity) * p.H;
    const int group = p.H / p.H_kv;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const int T_q = p.cu_q[p.batch], T_k = p.cu_k[p.batch];
        const int q_stride = p.H * D, kv_stride = p.H_kv * D;
        uint32_t q_issued = 0, k_issued = 0, v_issued = 0;
        bool ok = true;
        for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x) {
            const TileEntry te = p.tiles[idx / p.H];
            const int h = idx % p.H, hk = h / group;
            if (te.kt_hi <= te.kt_lo) continue;
            if (!(ok = mbar_wait_warp(q_empty, (q_issued & 1) ^ 1, abort_flag, &g_va_status))) break;
            load_tile<D>(smem + L::kQ, &tmQ, p.q, p.cu_q[te.b] + te.qt * kBlockM, T_q, q_stride,
                         h * D, q_full, lane);
            ++q_issued;
            const int k0 = p.cu_k[te.b];
            for (int kt = te.kt_lo; kt < te.kt_hi; ++kt) {
                const int s = k_issued % kStages;
                const uint32_t ph = (k_issued / kStages) & 1;
                if (!(ok = mbar_wait_warp(&k_empty[s], ph ^ 1, abort_flag, &g_va_status))) break;
                load_tile<D>(smem + L::kK + s * L::kTileBytes, &tmK, p.k, k0 + kt * kBlockN, T_k,
                             kv_stride, hk * D, &k_full[s], lane);
                ++k_issued;
                if (!(ok = mbar_wait_warp(&v_empty[s], ph ^ 1, abort_flag, &g_va_status))) break;
                load_tile<D>(smem + L::kV + s * L::kTileBytes, &tmV, p.v, k0 + kt * kBlockN, T_k,
                             kv_stride, hk * D, &v_full[s], lane);
                ++v_issued;
            }
        }
        if (!ok && lane == 0) {
            // abandoned: still wait (bounded) for the copies this warp issued
            // before the CTA releases its shared memory
            const unsigned long long t0 = global_timer_ns();
            auto drain = [&](uint64_t* bar, uint32_t issued_on_bar) {
                if (issued_on_bar == 0) return;
                while (!mbar_try_wait(bar, (issued_on_bar - 1) & 1) &&
                       global_timer_ns() - t0 < kWaitLimitNs) {
                }
            };
            drain(q_full, q_issued);
            for (int s = 0; s < kStages; ++s) {
                // loads into stage s: indices s, s + kStages, ...
                const uint32_t nk = k_issued > (uint32_t)s ? (k_issued - s + kStages - 1) / kStages : 0;
                const uint32_t nv = v_issued > (uint32_t)s ? (v_issued - s + kStages - 1) / kStages : 0;
                drain(&k_full[s], nk);
                drain(&v_full[s], nv);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kBlockN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            const uint32_t sQ = smem_u32(smem + L::kQ);
            const uint32_t sK = smem_u32(smem + L::kK);
            const uint32_t sV = smem_u32(smem + L::kV);
            uint32_t item_cnt = 0, kv_cnt = 0, tile_cnt = 0;
            bool ok = true;
            // O += P V for the tile with global counters (kv index, tile index)
            auto issue_pv = [&](uint32_t kv_i, uint32_t tile_i, bool first) -> bool {
                const uint32_t sb = tile_i & 1;
                if (!mbar_wait(&p_full[sb], (tile_i >> 1) & 1, abort_flag, &g_va_status)) return false;
                const int s = kv_i % kStages;
                if (!mbar_wait(&v_full[s], (kv_i / kStages) & 1, abort_flag, &g_va_status)) return false;
                tc_fence_after();
                const uint32_t vbase = sV + s * L::kTileBytes;
                const uint32_t pbase = tmem + (sb ? kTmemS1 : kTmemS0);
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    const uint64_t bdesc = smem_desc_sw128(vbase + kk * 16 * 128, L::kChunkBytes, 1024);
                    mma_ts(tmem + kTmemO, pbase + kk * 8, bdesc, idesc_pv, (!first || kk > 0) ? 1u : 0u);
                }
                mma_commit(o_done);
                mma_commit(&v_empty[s]);
                return true;
            };
            for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x) {
                const TileEntry te = p.tiles[idx / p.H];
                const int n = te.kt_hi - te.kt_lo;
                if (n <= 0) continue;
                if (!(ok = mbar_wait(q_full, item_cnt & 1, abort_flag, &g_va_status))) break;
                const uint32_t kv_base = kv_cnt, tile_base = tile_cnt;
                for (int j = 0; j < n; ++j) {
                    const uint32_t kv_i = kv_base + j, tile_i = tile_base + j;
                    const int s = kv_i % kStages;
                    if (!(ok = mbar_wait(&k_full[s], (kv_i / kStages) & 1, abort_flag, &g_va_status))) break;
                    tc_fence_after();
                    const uint32_t kbase = sK + s * L::kTileBytes;
                    const uint32_t sdst = tmem + ((tile_i & 1) ? kTmemS1 : kTmemS0);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * L::kChunkBytes + (kk & 3) * 32;
                        mma_ss(sdst, smem_desc_sw128(sQ + off, 16, 1024),
                               smem_desc_sw128(kbase + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&s_full[tile_i & 1]);
                    mma_commit(&k_empty[s]);
                    if (j == n - 1) mma_commit(q_empty);
                    if (j > 0 && !(ok = issue_pv(kv_i - 1, tile_i - 1, j - 1 == 0))) break;
                }
                if (!ok) break;
                if (!(ok = issue_pv(kv_base + n - 1, tile_base + n - 1, n == 1))) break;
                kv_cnt += n;
                tile_cnt += n;
                ++item_cnt;
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;          // query row within the tile
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t tile_cnt = 0, o_cnt = 0;
        bool ok = true;
        for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x) {
            const TileEntry te = p.tiles[idx / p.H];
            const int h = idx % p.H;
            const int L_q = p.cu_q[te.b + 1] - p.cu_q[te.b];
            const int L_k = p.cu_k[te.b + 1] - p.cu_k[te.b];
            const int i = te.qt * kBlockM + row;
            const bool row_valid = i < L_q;
            int lo, hi;
            row_key_interval(i, L_q, L_k, p.causal != 0, p.window, lo, hi);
            const size_t out_row = static_cast<size_t>(p.cu_q[te.b] + i) * p.H + h;
            const int n = te.kt_hi - te.kt_lo;
            if (n <= 0) {
                if (row_valid) {
                    uint4* o4 = reinterpret_cast<uint4*>(p.out + out_row * D);
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) o4[c] = make_uint4(0u, 0u, 0u, 0u);
                    p.lse[out_row] = -INFINITY;
                }
                continue;
            }
            float m_ref = -INFINITY, l = 0.f;
            for (int j = 0; j < n; ++j, ++tile_cnt) {
                const uint32_t sb = tile_cnt & 1;
                if (!(ok = mbar_wait_warp(&s_full[sb], (tile_cnt >> 1) & 1, abort_flag, &g_va_status))) break;
                __syncwarp();
                tc_fence_after();
                const uint32_t sbase = tmem + lane_addr + (sb ? kTmemS1 : kTmemS0);
                float s[kBlockN];
                {
                    // all four loads in flight before a single wait
                    uint32_t r0[32], r1[32], r2[32], r3[32];
                    tmem_ld32(sbase + 0, r0);
                    tmem_ld32(sbase + 32, r1);
                    tmem_ld32(sbase + 64, r2);
                    tmem_ld32(sbase + 96, r3);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        s[x] = __uint_as_float(r0[x]);
                        s[32 + x] = __uint_as_float(r1[x]);
                        s[64 + x] = __uint_as_float(r2[x]);
                        s[96 + x] = __uint_as_float(r3[x]);
                    }
                }
                const int key0 = (te.kt_lo + j) * kBlockN;
                const bool full_tile = lo <= key0 && key0 + kBlockN - 1 <= hi;
                if (__any_sync(0xffffffffu, !full_tile)) {
#pragma unroll
                    for (int c = 0; c < kBlockN; ++c) {
                        const int kj = key0 + c;
                        s[c] = (kj >= lo && kj <= hi) ? s[c] : -INFINITY;
                    }
                }
                // row max as a tree (short dependency chains)
                float mv[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) mv[x] = s[x];
#pragma unroll
                for (int c = 8; c < kBlockN; c += 8)
#pragma unroll
                    for (int x = 0; x < 8; ++x) mv[x] = fmaxf(mv[x], s[c + x]);
                const float mx = fmaxf(fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3])),
                                       fmaxf(fmaxf(mv[4], mv[5]), fmaxf(mv[6], mv[7])));
                const float m_tile = mx * p.scale_log2;  // -inf stays -inf
                const float m_cand = fmaxf(m_ref, m_tile);
                const bool want = (j == 0) || (m_cand > m_ref + kRescaleThreshold);
                const bool move = __any_sync(0xffffffffu, want);
                float alpha = 1.f;
                if (move) {
                    alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - m_cand);
                    m_ref = m_cand;
                }
                const float m_sub = (m_ref == -INFINITY) ? 0.f : m_ref;
                float sums[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                uint32_t pk[kBlockN / 2];
#pragma unroll
                for (int c = 0; c < kBlockN; c += 2) {
                    const float p0 = ex2_approx(fmaf(s[c], p.scale_log2, -m_sub));
                    const float p1 = ex2_approx(fmaf(s[c + 1], p.scale_log2, -m_sub));
                    sums[(c >> 1) & 7] += p0 + p1;
                    pk[c / 2] = pack_bf16x2(p0, p1);
                }
                const float rowsum = ((sums[0] + sums[1]) + (sums[2] + sums[3])) +
                                     ((sums[4] + sums[5]) + (sums[6] + sums[7]));
                l = l * alpha + rowsum;
                if (j > 0) {
                    // O must hold P_{j-1} V_{j-1} before it is rescaled
                    if (!(ok = mbar_wait_warp(o_done, o_cnt & 1, abort_flag, &g_va_status))) break;
                    ++o_cnt;
                    __syncwarp();
                    tc_fence_after();
                    if (move) {
                        const uint32_t obase = tmem + lane_addr + kTmemO;
#pragma unroll
                        for (int c = 0; c < D / 32; c += 2) {
                            uint32_t r[32], r2[32];
                            tmem_ld32(obase + c * 32, r);
                            tmem_ld32(obase + (c + 1) * 32, r2);
                            tmem_wait_ld();
#pragma unroll
                            for (int x = 0; x < 32; ++x) {
                                r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
                                r2[x] = __float_as_uint(__uint_as_float(r2[x]) * alpha);
                            }
                            tmem_st32(obase + c * 32, r);
                            tmem_st32(obase + (c + 1) * 32, r2);
                        }
                    }
                }
                {
                    uint32_t r0[32], r1[32];
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        r0[x] = pk[x];
                        r1[x] = pk[32 + x];
                    }
                    tmem_st32(sbase, r0);
                    tmem_st32(sbase + 32, r1);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sb]);
            }
            if (!ok) break;
            // epilogue: wait for the last P V, then O / l and logsumexp
            if (!(ok = mbar_wait_warp(o_done, o_cnt & 1, abort_flag, &g_va_status))) break;
            ++o_cnt;
            __syncwarp();
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            const uint32_t obase = tmem + lane_addr + kTmemO;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(obase + c * 32, r);
                tmem_wait_ld();
                if (row_valid) {
                    uint4* o4 = reinterpret_cast<uint4*>(p.out + out_row * D + c * 32);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(r[8 * x + 0]) * inv_l, __uint_as_float(r[8 * x + 1]) * inv_l);
                        w.y = pack_bf16x2(__uint_as_float(r[8 * x + 2]) * inv_l, __uint_as_float(r[8 * x + 3]) * inv_l);
                        w.z = pack_bf16x2(__uint_as_float(r[8 * x + 4]) * inv_l, __uint_as_float(r[8 * x + 5]) * inv_l);
                        w.w = pack_bf16x2(__uint_as_float(r[8 * x + 6]) * inv_l, __uint_as_float(r[8 * x + 7]) * inv_l);
                        o4[x] = w;
                    }
                }
            }
            if (row_valid) {
                p.lse[out_row] = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994530942f : -INFINITY;
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace va
