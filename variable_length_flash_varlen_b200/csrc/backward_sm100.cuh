// Packed variable-length attention backward for sm_100a: dq, dk, dv of
// VarLenAttentionOps::varlen_attention_bwd (boostr 0.2.0 varlen_attention.rs:
// dk and dv are [total_k, num_kv_heads, D] under GQA, summed over the query
// heads that share a KV head), consuming the forward's logsumexp (boostr
// flash.rs, FlashAttentionOps docs: "logsumexp (F32, for backward pass)").
//
// With s_ij = q_i.k_j / sqrt(D) on the visible (i, j) pairs, P_ij =
// exp(s_ij - lse_i), dP_ij = dout_i.v_j and Delta_i = dout_i.out_i:
//   dS_ij = P_ij (dP_ij - Delta_i)
//   dv_j = sum_i P_ij dout_i,  dk_j = sum_i dS_ij q_i / sqrt(D),
//   dq_i = sum_j dS_ij k_j / sqrt(D).
// Three kernels, no atomics, every output element written by one CTA:
//   bwd_delta_kernel   Delta_i (one warp per token row and head)
//   bwd_dkdv_kernel    one CTA per (key tile of 128 keys, KV head, sequence):
//                      K and V stay in shared memory; for every query head of
//                      the group and every 128-row query tile that sees the key
//                      tile: S^T = K Q^T and dP^T = V dout^T on tensor cores,
//                      P^T and dS^T (bf16) back into tensor memory, then
//                      dV += P^T dout and dK += dS^T Q (TS form), accumulated
//                      in tensor memory over the whole loop
//   bwd_dq_kernel      one CTA per (128-row query tile, query head, sequence):
//                      Q and dout stay; for every visible key tile S = Q K^T,
//                      dP = dout V^T, dS (bf16) into tensor memory, dQ += dS K
// Warp roles (192 threads): warps 0-3 the element-wise work and the epilogue
// (one key row, or one query row, per thread), warp 4 the TMA producer, warp 5
// the tensor-memory owner and MMA issuer (one lane).
#pragma once

#include "prefill_sm100.cuh"

namespace va {

constexpr int kBwdThreads = 192;
constexpr int kBwdLoadWarp = 4;
constexpr int kBwdMmaWarp = 5;

struct BwdParams {
    const int* cu_q;
    const int* cu_k;
    int batch, H, H_kv, causal, window;
    const uint8_t* q;     // bf16 bytes, [total_q, H, D]
    const uint8_t* k;     // [total_k, H_kv, D]
    const uint8_t* v;
    const uint8_t* dout;  // [total_q, H, D]
    const uint8_t* out;   // forward output, [total_q, H, D]
    const float* lse;     // forward logsumexp (natural log), [total_q, H]
    float* delta;         // [total_q, H] written by bwd_delta_kernel
    uint8_t* dq;          // bf16 outputs
    uint8_t* dk;
    uint8_t* dv;
    float scale_log2;     // log2(e) / sqrt(D)
    float scale;          // 1 / sqrt(D)
};

// Q and dout as [rows][H * D], K and V as [rows][H_kv * D]: 128-row boxes and
// 8-row boxes for a tile that runs past the end of the packed tensor.
struct BwdMaps {
    CUtensorMap q, dout, k, v;
    CUtensorMap q8, dout8, k8, v8;
};

// Delta_i = sum_d dout[i, d] * out[i, d] in f32, one warp per (token, head) row.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const BwdParams p) {
    const long long rows = static_cast<long long>(p.cu_q[p.batch]) * p.H;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31;
    constexpr int kPer = D / 32;  // bf16 values per lane
    const __nv_bfloat16* o = reinterpret_cast<const __nv_bfloat16*>(p.out) + row * D + lane * kPer;
    const __nv_bfloat16* g = reinterpret_cast<const __nv_bfloat16*>(p.dout) + row * D + lane * kPer;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc = fmaf(__bfloat162float(o[e]), __bfloat162float(g[e]), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) p.delta[row] = acc;
}

template <int D>
struct BwdSmem {
    using T = PrefillSmem<D, ElemBf16>;
    static constexpr int kTile = T::kTileBytes;  // 128 rows x D bf16, 128-byte swizzle
    // dK/dV kernel: K, V once; Q, dout, base-2 lse and Delta double-buffered
    // dQ kernel:   Q, dout once; K, V double-buffered
    static constexpr int kFixed0 = 0;
    static constexpr int kFixed1 = kTile;
    static constexpr int kRing0 = 2 * kTile;      // [2]
    static constexpr int kRing1 = 4 * kTile;      // [2]
    static constexpr int kRows = 6 * kTile;       // [2][128] f32 lse * log2(e), [2][128] f32 Delta
    static constexpr int kBar = kRows + 4 * 128 * 4;
    // fixed_full, ring_full[2], ring_empty[2], s_full, p_ready, acc_done
    static constexpr int kNumBars = 8;
    static constexpr int kMisc = kBar + kNumBars * 8;  // tmem slot, abort flag
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = (kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024;
    static_assert(kAlloc <= 232448, "beyond the 227 KB of shared memory a CTA may use");
};

// Per-role state shared by the two tile kernels.
struct BwdBars {
    uint64_t* fixed_full;
    uint64_t* ring_full;   // [2]
    uint64_t* ring_empty;  // [2]
    uint64_t* s_full;
    uint64_t* p_ready;
    uint64_t* acc_done;
    uint32_t* tmem_slot;
    volatile int* abort_flag;
};

template <int D>
__device__ __forceinline__ BwdBars bwd_setup(uint8_t* smem, int warp) {
    using L = BwdSmem<D>;
    BwdBars r;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    r.fixed_full = bars;
    r.ring_full = bars + 1;
    r.ring_empty = bars + 3;
    r.s_full = bars + 5;
    r.p_ready = bars + 6;
    r.acc_done = bars + 7;
    r.tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    r.abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    if (threadIdx.x == 0) {
        mbar_init(r.fixed_full, 2);  // two tile loads
        for (int s = 0; s < 2; ++s) {
            mbar_init(&r.ring_full[s], 2);
            mbar_init(&r.ring_empty[s], 1);
        }
        mbar_init(r.s_full, 1);
        mbar_init(r.p_ready, 4);  // the four element-wise warps
        mbar_init(r.acc_done, 1);
        *r.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(r.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return r;
}

template <int D>
__device__ __forceinline__ void bwd_teardown(const BwdBars& r, uint32_t tmem, int warp) {
    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Producer's bounded wait, on giving up, for the copies it issued on `bar`.
__device__ __forceinline__ void bwd_drain(uint64_t* bar, uint32_t issued, unsigned long long t0) {
    if (issued == 0) return;
    while (!mbar_try_wait(bar, (issued - 1) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
}

// This thread's row (its TMEM lane) of a D-column f32 accumulator at tensor
// memory address `taddr`, scaled by `mul`, as bf16 to dst + row * row_pitch
// (nothing is stored when !valid; the loads still run, they are warp-wide).
template <int D>
__device__ __forceinline__ void bwd_store_rows(uint32_t taddr, float mul, uint8_t* dst,
                                               long long row_pitch, int row, bool valid) {
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_wait_ld();
        if (valid) {
            uint4* o = reinterpret_cast<uint4*>(dst + row * row_pitch + c * 64);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(r[8 * e + 0]) * mul, __uint_as_float(r[8 * e + 1]) * mul);
                w.y = pack_bf16x2(__uint_as_float(r[8 * e + 2]) * mul, __uint_as_float(r[8 * e + 3]) * mul);
                w.z = pack_bf16x2(__uint_as_float(r[8 * e + 4]) * mul, __uint_as_float(r[8 * e + 5]) * mul);
                w.w = pack_bf16x2(__uint_as_float(r[8 * e + 6]) * mul, __uint_as_float(r[8 * e + 7]) * mul);
                o[e] = w;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// dK, dV: one CTA per (key tile kt, KV head hk, sequence b) = blockIdx (x, y, z).
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ BwdMaps maps, const BwdParams p) {
    using L = BwdSmem<D>;
    using T = PrefillSmem<D, ElemBf16>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kt = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int G = p.H / p.H_kv;
    const int cq = p.cu_q[b], ck = p.cu_k[b];
    const int L_q = p.cu_q[b + 1] - cq, L_k = p.cu_k[b + 1] - ck;
    const int k0 = kt * kBlockN;
    if (k0 >= L_k) return;  // the whole CTA, before any barrier
    const int k_last = min(L_k, k0 + kBlockN) - 1;
    const int delta_k = L_k - L_q;
    // query rows that see a key of [k0, k_last] (bottom-right causal, window of
    // W keys ending at the diagonal): i >= k0 - delta_k, i <= k_last - delta_k + W - 1
    int r0 = 0, r1 = L_q - 1;
    if (p.causal || p.window > 0) r0 = max(0, k0 - delta_k);
    if (p.window > 0) r1 = min(r1, k_last - delta_k + p.window - 1);
    const int n_qt = (L_q > 0 && r1 >= r0) ? r1 / kBlockM - r0 / kBlockM + 1 : 0;
    const int qt0 = r0 / kBlockM;
    const int n_steps = G * n_qt;
    const long long kv_pitch = static_cast<long long>(p.H_kv) * D * 2;
    if (n_steps == 0) {
        // no query sees these keys: their gradients are zero
        for (int idx = threadIdx.x; idx < (k_last - k0 + 1) * (D / 8); idx += blockDim.x) {
            const int r = idx / (D / 8), c = idx % (D / 8);
            const long long off = (static_cast<long long>(ck) + k0 + r) * kv_pitch + hk * D * 2 + c * 16;
            *reinterpret_cast<uint4*>(p.dk + off) = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(p.dv + off) = make_uint4(0u, 0u, 0u, 0u);
        }
        return;
    }

    const BwdBars bar = bwd_setup<D>(smem, warp);
    const uint32_t tmem = *bar.tmem_slot;
    unsigned* status = &g_va_status;
    float* lse_s = reinterpret_cast<float*>(smem + L::kRows);            // [2][128]
    float* dlt_s = reinterpret_cast<float*>(smem + L::kRows + 1024);     // [2][128]
    constexpr uint32_t kS = 0, kDP = 128, kDV = 256, kDK = 256 + D;      // tensor-memory columns

    if (warp == kBwdLoadWarp) {
        // ------------------------------------------------------------ producer
        const int T_q = p.cu_q[p.batch], T_k = p.cu_k[p.batch];
        const int q_stride = p.H * D * 2, kv_stride = p.H_kv * D * 2;
        uint32_t issued[2] = {0, 0};
        bool ok = true;
        load_tile<D, ElemBf16>(smem + L::kFixed0, &maps.k, &maps.k8, p.k, ck + k0, T_k, kv_stride,
                               hk * D, bar.fixed_full, lane);
        load_tile<D, ElemBf16>(smem + L::kFixed1, &maps.v, &maps.v8, p.v, ck + k0, T_k, kv_stride,
                               hk * D, bar.fixed_full, lane);
        for (int n = 0; n < n_steps; ++n) {
            const int st = n & 1;
            const int h = hk * G + n / n_qt, qt = qt0 + n % n_qt;
            if (!(ok = mbar_wait_warp(&bar.ring_empty[st], ((n >> 1) & 1) ^ 1, bar.abort_flag, status)))
                break;
            for (int r = lane; r < kBlockM; r += 32) {
                const int i = qt * kBlockM + r;
                float l2 = 0.f, dl = 0.f;  // rows past the sequence: masked, any finite value
                if (i < L_q) {
                    const float l = p.lse[static_cast<size_t>(cq + i) * p.H + h];
                    l2 = l == -INFINITY ? 0.f : l * 1.4426950408889634f;
                    dl = p.delta[static_cast<size_t>(cq + i) * p.H + h];
                }
                lse_s[st * kBlockM + r] = l2;
                dlt_s[st * kBlockM + r] = dl;
            }
            __syncwarp();
            load_tile<D, ElemBf16>(smem + L::kRing0 + st * L::kTile, &maps.q, &maps.q8, p.q,
                                   cq + qt * kBlockM, T_q, q_stride, h * D, &bar.ring_full[st], lane);
            load_tile<D, ElemBf16>(smem + L::kRing1 + st * L::kTile, &maps.dout, &maps.dout8, p.dout,
                                   cq + qt * kBlockM, T_q, q_stride, h * D, &bar.ring_full[st], lane);
            ++issued[st];
        }
        if (!ok && lane == 0) {
            const unsigned long long t0 = global_timer_ns();
            bwd_drain(bar.fixed_full, 1, t0);
            bwd_drain(&bar.ring_full[0], issued[0], t0);
            bwd_drain(&bar.ring_full[1], issued[1], t0);
        }
    } else if (warp == kBwdMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_ss = idesc_bf16_f32(128, kBlockM, false);
            constexpr uint32_t idesc_ts = idesc_bf16_f32(128, D, true);
            const uint64_t dk_ = smem_desc_sw128(smem_u32(smem + L::kFixed0), 16, 1024);
            const uint64_t dv_ = smem_desc_sw128(smem_u32(smem + L::kFixed1), 16, 1024);
            const uint64_t dq_k = smem_desc_sw128(smem_u32(smem + L::kRing0), 16, 1024);
            const uint64_t dd_k = smem_desc_sw128(smem_u32(smem + L::kRing1), 16, 1024);
            const uint64_t dq_mn = smem_desc_sw128(smem_u32(smem + L::kRing0), T::kChunkBytes, 1024);
            const uint64_t dd_mn = smem_desc_sw128(smem_u32(smem + L::kRing1), T::kChunkBytes, 1024);
            const uint32_t hi_k = static_cast<uint32_t>(dk_ >> 32), hi_mn = static_cast<uint32_t>(dq_mn >> 32);
            bool ok = mbar_wait(bar.fixed_full, 0, bar.abort_flag, status);
            tc_fence_after();
            for (int n = 0; n < n_steps && ok; ++n) {
                const int st = n & 1;
                if (!(ok = mbar_wait(&bar.ring_full[st], (n >> 1) & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                const uint32_t ring = (st * L::kTile) >> 4;
                // S^T = K Q^T and dP^T = V dout^T (K-major operands, K = D)
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * T::kChunkBytes + (kk & 3) * 32) >> 4;
                    mma_ss_lh<idesc_ss>(tmem + kS, static_cast<uint32_t>(dk_) + off, hi_k,
                                        static_cast<uint32_t>(dq_k) + ring + off, hi_k, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * T::kChunkBytes + (kk & 3) * 32) >> 4;
                    mma_ss_lh<idesc_ss>(tmem + kDP, static_cast<uint32_t>(dv_) + off, hi_k,
                                        static_cast<uint32_t>(dd_k) + ring + off, hi_k, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar.s_full);
                if (!(ok = mbar_wait(bar.p_ready, n & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                // dV += P^T dout and dK += dS^T Q (A from tensor memory, B MN-major, K = 128 rows)
#pragma unroll
                for (int kk = 0; kk < kBlockM / 16; ++kk) {
                    const uint32_t boff = ring + ((kk * 16 * 128) >> 4);
                    const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
                    mma_ts_lh<idesc_ts>(tmem + kDV, tmem + kS + kk * 8,
                                        static_cast<uint32_t>(dd_mn) + boff, hi_mn, acc);
                    mma_ts_lh<idesc_ts>(tmem + kDK, tmem + kDP + kk * 8,
                                        static_cast<uint32_t>(dq_mn) + boff, hi_mn, acc);
                }
                mma_commit(&bar.ring_empty[st]);
            }
            mma_commit(bar.acc_done);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ element-wise
        const int quarter = warp & 3;
        const int jj = quarter * 32 + lane;                 // key row of the tile (TMEM lane)
        const int j = k0 + jj;                              // key index in the sequence
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        // query rows that see key j: [i_lo, i_hi] (empty when j is past the keys)
        int i_lo = 0, i_hi = L_q - 1;
        if (p.causal || p.window > 0) i_lo = max(0, j - delta_k);
        if (p.window > 0) i_hi = min(i_hi, j - delta_k + p.window - 1);
        if (j >= L_k) i_hi = -1;
        const unsigned i_span = i_hi >= i_lo ? static_cast<unsigned>(i_hi - i_lo) : 0u;
        const int i_base = i_hi >= i_lo ? i_lo : (1 << 30);
        bool ok = true;
        for (int n = 0; n < n_steps; ++n) {
            const int st = n & 1;
            const int qt = qt0 + n % n_qt;
            if (!(ok = mbar_wait_warp(bar.s_full, n & 1, bar.abort_flag, status))) break;
            // the producer's stores of this step's logsumexp and Delta rows are
            // released by its arrival on ring_full (already complete: the MMA
            // warp waited for it before the products this wait observed)
            if (!(ok = mbar_wait_warp(&bar.ring_full[st], (n >> 1) & 1, bar.abort_flag, status))) break;
            tc_fence_after();
            const float* l2 = lse_s + st * kBlockM;
            const float* dl = dlt_s + st * kBlockM;
#pragma unroll 1
            for (int c = 0; c < kBlockM / 32; ++c) {
                uint32_t sr[32], dr[32];
                tmem_ld32(tmem + lane_addr + kS + c * 32, sr);
                tmem_ld32(tmem + lane_addr + kDP + c * 32, dr);
                tmem_wait_ld();
                uint32_t pk[16], dk16[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float pv[2], dsv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int col = c * 32 + e + u;
                        const int i = qt * kBlockM + col;
                        const bool vis = static_cast<unsigned>(i - i_base) <= i_span;
                        const float pe = vis ? ex2_approx(fmaf(__uint_as_float(sr[e + u]), p.scale_log2, -l2[col]))
                                             : 0.f;
                        pv[u] = pe;
                        dsv[u] = pe * (__uint_as_float(dr[e + u]) - dl[col]);
                    }
                    pk[e / 2] = pack_bf16x2(pv[0], pv[1]);
                    dk16[e / 2] = pack_bf16x2(dsv[0], dsv[1]);
                }
                // P^T and dS^T over the S^T / dP^T columns this and earlier chunks have read
                tmem_st16(tmem + lane_addr + kS + c * 16, pk);
                tmem_st16(tmem + lane_addr + kDP + c * 16, dk16);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.p_ready);
        }
        if (ok) ok = mbar_wait_warp(bar.acc_done, 0, bar.abort_flag, status);
        if (ok) {
            tc_fence_after();
            const bool valid = j < L_k;
            uint8_t* base_v = p.dv + (static_cast<long long>(ck) + k0) * kv_pitch + hk * D * 2;
            uint8_t* base_k = p.dk + (static_cast<long long>(ck) + k0) * kv_pitch + hk * D * 2;
            bwd_store_rows<D>(tmem + lane_addr + kDV, 1.f, base_v, kv_pitch, jj, valid);
            bwd_store_rows<D>(tmem + lane_addr + kDK, p.scale, base_k, kv_pitch, jj, valid);
        }
    }
    bwd_teardown<D>(bar, tmem, warp);
}

// ---------------------------------------------------------------------------
// dQ: one CTA per (query tile qt, query head h, sequence b) = blockIdx (x, y, z).
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dq_kernel(const __grid_constant__ BwdMaps maps, const BwdParams p) {
    using L = BwdSmem<D>;
    using T = PrefillSmem<D, ElemBf16>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / (p.H / p.H_kv);
    const int cq = p.cu_q[b], ck = p.cu_k[b];
    const int L_q = p.cu_q[b + 1] - cq, L_k = p.cu_k[b + 1] - ck;
    const int q0 = qt * kBlockM;
    if (q0 >= L_q) return;  // the whole CTA, before any barrier
    int kt_lo, kt_hi;
    rows_key_range(q0, kBlockM, L_q, L_k, p.causal != 0, p.window, kt_lo, kt_hi);
    const int n_steps = kt_hi - kt_lo;
    const long long q_pitch = static_cast<long long>(p.H) * D * 2;
    if (n_steps <= 0) {
        // these rows see no key: dq is zero
        const int rows = min(L_q - q0, kBlockM);
        for (int idx = threadIdx.x; idx < rows * (D / 8); idx += blockDim.x) {
            const int r = idx / (D / 8), c = idx % (D / 8);
            *reinterpret_cast<uint4*>(p.dq + (static_cast<long long>(cq) + q0 + r) * q_pitch + h * D * 2 +
                                      c * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        return;
    }

    const BwdBars bar = bwd_setup<D>(smem, warp);
    const uint32_t tmem = *bar.tmem_slot;
    unsigned* status = &g_va_status;
    constexpr uint32_t kS = 0, kDP = 128, kDQ = 256;  // tensor-memory columns

    if (warp == kBwdLoadWarp) {
        // ------------------------------------------------------------ producer
        const int T_q = p.cu_q[p.batch], T_k = p.cu_k[p.batch];
        const int q_stride = p.H * D * 2, kv_stride = p.H_kv * D * 2;
        uint32_t issued[2] = {0, 0};
        bool ok = true;
        load_tile<D, ElemBf16>(smem + L::kFixed0, &maps.q, &maps.q8, p.q, cq + q0, T_q, q_stride, h * D,
                               bar.fixed_full, lane);
        load_tile<D, ElemBf16>(smem + L::kFixed1, &maps.dout, &maps.dout8, p.dout, cq + q0, T_q, q_stride,
                               h * D, bar.fixed_full, lane);
        for (int n = 0; n < n_steps; ++n) {
            const int st = n & 1, kt = kt_lo + n;
            if (!(ok = mbar_wait_warp(&bar.ring_empty[st], ((n >> 1) & 1) ^ 1, bar.abort_flag, status)))
                break;
            load_tile<D, ElemBf16>(smem + L::kRing0 + st * L::kTile, &maps.k, &maps.k8, p.k,
                                   ck + kt * kBlockN, T_k, kv_stride, hk * D, &bar.ring_full[st], lane);
            load_tile<D, ElemBf16>(smem + L::kRing1 + st * L::kTile, &maps.v, &maps.v8, p.v,
                                   ck + kt * kBlockN, T_k, kv_stride, hk * D, &bar.ring_full[st], lane);
            ++issued[st];
        }
        if (!ok && lane == 0) {
            const unsigned long long t0 = global_timer_ns();
            bwd_drain(bar.fixed_full, 1, t0);
            bwd_drain(&bar.ring_full[0], issued[0], t0);
            bwd_drain(&bar.ring_full[1], issued[1], t0);
        }
    } else if (warp == kBwdMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_ss = idesc_bf16_f32(128, kBlockN, false);
            constexpr uint32_t idesc_ts = idesc_bf16_f32(128, D, true);
            const uint64_t dq_ = smem_desc_sw128(smem_u32(smem + L::kFixed0), 16, 1024);
            const uint64_t dd_ = smem_desc_sw128(smem_u32(smem + L::kFixed1), 16, 1024);
            const uint64_t dk_k = smem_desc_sw128(smem_u32(smem + L::kRing0), 16, 1024);
            const uint64_t dv_k = smem_desc_sw128(smem_u32(smem + L::kRing1), 16, 1024);
            const uint64_t dk_mn = smem_desc_sw128(smem_u32(smem + L::kRing0), T::kChunkBytes, 1024);
            const uint32_t hi_k = static_cast<uint32_t>(dq_ >> 32), hi_mn = static_cast<uint32_t>(dk_mn >> 32);
            bool ok = mbar_wait(bar.fixed_full, 0, bar.abort_flag, status);
            tc_fence_after();
            for (int n = 0; n < n_steps && ok; ++n) {
                const int st = n & 1;
                if (!(ok = mbar_wait(&bar.ring_full[st], (n >> 1) & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                const uint32_t ring = (st * L::kTile) >> 4;
                // S = Q K^T and dP = dout V^T (K-major operands, K = D)
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * T::kChunkBytes + (kk & 3) * 32) >> 4;
                    mma_ss_lh<idesc_ss>(tmem + kS, static_cast<uint32_t>(dq_) + off, hi_k,
                                        static_cast<uint32_t>(dk_k) + ring + off, hi_k, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * T::kChunkBytes + (kk & 3) * 32) >> 4;
                    mma_ss_lh<idesc_ss>(tmem + kDP, static_cast<uint32_t>(dd_) + off, hi_k,
                                        static_cast<uint32_t>(dv_k) + ring + off, hi_k, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar.s_full);
                if (!(ok = mbar_wait(bar.p_ready, n & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                // dQ += dS K (A from tensor memory, B = K MN-major, K = 128 keys)
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    mma_ts_lh<idesc_ts>(tmem + kDQ, tmem + kDP + kk * 8,
                                        static_cast<uint32_t>(dk_mn) + ring + ((kk * 16 * 128) >> 4), hi_mn,
                                        (n > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bar.ring_empty[st]);
            }
            mma_commit(bar.acc_done);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ element-wise
        const int quarter = warp & 3;
        const int ii = quarter * 32 + lane;  // query row of the tile (TMEM lane)
        const int i = q0 + ii;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const bool row_valid = i < L_q;
        float l2 = 0.f, dl = 0.f;
        int lo = 0, hi = -1;
        if (row_valid) {
            const float l = p.lse[static_cast<size_t>(cq + i) * p.H + h];
            l2 = l == -INFINITY ? 0.f : l * 1.4426950408889634f;
            dl = p.delta[static_cast<size_t>(cq + i) * p.H + h];
            row_key_interval(i, L_q, L_k, p.causal != 0, p.window, lo, hi);
        }
        const unsigned span = hi >= lo ? static_cast<unsigned>(hi - lo) : 0u;
        const int base = hi >= lo ? lo : (1 << 30);
        bool ok = true;
        for (int n = 0; n < n_steps; ++n) {
            const int kt = kt_lo + n;
            if (!(ok = mbar_wait_warp(bar.s_full, n & 1, bar.abort_flag, status))) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < kBlockN / 32; ++c) {
                uint32_t sr[32], dr[32];
                tmem_ld32(tmem + lane_addr + kS + c * 32, sr);
                tmem_ld32(tmem + lane_addr + kDP + c * 32, dr);
                tmem_wait_ld();
                uint32_t dk16[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float dsv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int jkey = kt * kBlockN + c * 32 + e + u;
                        const bool vis = static_cast<unsigned>(jkey - base) <= span;
                        const float pe = vis ? ex2_approx(fmaf(__uint_as_float(sr[e + u]), p.scale_log2, -l2)) : 0.f;
                        dsv[u] = pe * (__uint_as_float(dr[e + u]) - dl);
                    }
                    dk16[e / 2] = pack_bf16x2(dsv[0], dsv[1]);
                }
                // dS over the dP columns this and earlier chunks have read
                tmem_st16(tmem + lane_addr + kDP + c * 16, dk16);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.p_ready);
        }
        if (ok) ok = mbar_wait_warp(bar.acc_done, 0, bar.abort_flag, status);
        if (ok) {
            tc_fence_after();
            uint8_t* base_q = p.dq + (static_cast<long long>(cq) + q0) * q_pitch + h * D * 2;
            bwd_store_rows<D>(tmem + lane_addr + kDQ, p.scale, base_q, q_pitch, ii, row_valid);
        }
    }
    bwd_teardown<D>(bar, tmem, warp);
}

}  // namespace va
