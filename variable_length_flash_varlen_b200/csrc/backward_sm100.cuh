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
// Two persistent kernels, no atomics, every output element written by one
// CTA, dQ first.  Each works through a device-built list of its tiles,
// longest first, claimed from a grid-wide counter (one CTA per SM):
//   bwd_dq_kernel      item = (128-row query tile, query head, sequence):
//                      Delta_i of its rows (stored for the other kernel), then
//                      with Q and dout resident, for every visible key tile
//                      S = Q K^T, dP = dout V^T, dS (bf16) into tensor memory,
//                      dQ += dS K
//   bwd_dkdv_kernel    item = (key tile of 128 keys, KV head, sequence):
//                      K and V stay in shared memory; for every query head of
//                      the group and every 128-row query tile that sees the key
//                      tile: S^T = K Q^T, P^T (bf16, in registers) while dP^T =
//                      V dout^T runs, then dS^T, both stored (bf16) over the dP^T
//                      columns, then dV += P^T dout and dK += dS^T Q (TS form),
//                      the two accumulators in tensor memory over the whole
//                      loop; the next S^T runs as soon as S^T has been read
// The streamed tiles come through two rings: ring 0 (K for dQ, Q for dK/dV,
// three stages: its last reader ends a step, the next-but-one step's first
// product starts the next) and ring 1 (V, or dout with its step's lse and
// Delta, two stages).  An item's resident tiles are reloaded once its last
// products that read them (its last S and dP) are done, its accumulators read
// out by the element-wise warps before the next item's first product
// overwrites them; the products of one item's steps and the barrier phases run
// on across items.
// Warp roles (320 threads): warps 0-7 the element-wise work and the epilogue
// (one key row, or one query row, per thread; warps w and w + 4 share a
// tensor-memory lane quarter and take one half of the 128 columns each), warp
// 8 the TMA producer, warp 9 the tensor-memory owner and MMA issuer (one lane).
#pragma once

#include "prefill_sm100.cuh"

namespace va {

// Status bit of the backward kernels (next to the bits of ptx.cuh): a kernel
// whose layout needs a 1024-byte-aligned shared-memory base found it misaligned.
constexpr unsigned kStatusSmemAlign = 4u;

constexpr int kBwdThreads = 320;
constexpr int kBwdEwWarps = 8;
constexpr int kBwdLoadWarp = 8;
constexpr int kBwdMmaWarp = 9;

// Where the bf16 values formed from 32-column chunk c of an f32 tile (S^T,
// dP^T, S or dP, 128 columns) are stored: the two warps of a lane quarter
// own chunks {0, 1} and {2, 3}, and each writes only over columns it has
// already read itself (16 packed columns per chunk, at 0, 16 and 64, 80).
__host__ __device__ constexpr uint32_t bwd_pcol(int c) { return (c >> 1) * 64 + (c & 1) * 16; }
// The same place seen by the MMA that consumes it: 16 rows of K per step.
__host__ __device__ constexpr uint32_t bwd_kcol(int kk) { return bwd_pcol(kk >> 1) + (kk & 1) * 8; }

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
    // per (head, token): {lse * log2(e), Delta}, head-major [H][rows_cap], written by
    // bwd_dq_kernel for every query row that sees a key, read by bwd_dkdv_kernel
    // (128 consecutive rows of one head per query tile)
    float2* rowinfo;
    long long rows_cap;   // >= total_q

    uint8_t* dq;          // bf16 outputs
    uint8_t* dk;
    uint8_t* dv;
    float scale_log2;     // log2(e) / sqrt(D)
    float scale;          // 1 / sqrt(D)
    // work lists (build_bwd_list_kernel): query tiles for dQ, key tiles for dK/dV
    const TileEntry* list_q;
    SchedHeader* hdr_q;
    int cap_q;
    const TileEntry* list_k;
    SchedHeader* hdr_k;
    int cap_k;
};

// A claimed work item as the producer publishes it to the other roles.
struct BwdItem {
    int idx;                // item index (entry x heads + head), -1 = no more work
    int b, tile, a0, a1;    // the list entry
    int head;
    int pad[2];
};

// Q and dout as [rows][H * D], K and V as [rows][H_kv * D]: 128-row boxes and
// 8-row boxes for a tile that runs past the end of the packed tensor.
struct BwdMaps {
    CUtensorMap q, dout, k, v;
    CUtensorMap q8, dout8, k8, v8;
};

template <int D, bool kDq>
struct BwdSmem {
    using T = PrefillSmem<D, ElemBf16>;
    static constexpr int kTile = T::kTileBytes;  // 128 rows x D bf16, 128-byte swizzle
    // Ring 0 has three stages: its tile's last reader (dQ, or dK) ends a step
    // while the next-but-one step's first product (S, or S^T) starts the next.
    // dK/dV kernel: K, V once; Q in ring 0; dout in ring 1 (two stages) with
    //               the base-2 lse and Delta of its step
    // dQ kernel:   Q, dout once; K in ring 0; V in ring 1 (two stages: read by
    //               dP only, early in a step)
    static constexpr int kStages0 = 3;
    static constexpr int kFixed0 = 0;
    static constexpr int kFixed1 = kTile;
    static constexpr int kRing0 = 2 * kTile;                  // [kStages0]
    static constexpr int kRing1 = kRing0 + kStages0 * kTile;  // [2]
    static constexpr int kRows = kRing1 + 2 * kTile;          // dK/dV: [2][128] f32 lse * log2(e), [2][128] f32 Delta
    static constexpr int kBar = kRows + (kDq ? 0 : 4 * 128 * 4);
    // fixed_full, ring_full[3], ring_empty[3], s_full, p_ready, acc_done, dp_full, ds_ready,
    // p_read, fixed_empty, acc_free, item_full[2], item_empty[2], ring1_full[2], ring1_empty[2]
    static constexpr int kNumBars = 23;
    static constexpr int kMisc = kBar + kNumBars * 8;  // tmem slot, abort flag
    static constexpr int kItems = kMisc + 16;          // BwdItem [2]
    static constexpr int kBytes = kItems + 2 * 32;
    // 1 KB of slack aligns the layout to 1024 bytes inside any base; a layout
    // too large for the slack relies on the base itself being aligned (the
    // kernel checks, and on a misaligned base raises kStatusSmemAlign and
    // returns before any access)
    static constexpr bool kNeedsAlignedBase = kBytes + 1024 > 232448;
    static constexpr int kAlloc =
        kNeedsAlignedBase ? kBytes : ((kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024);
    static_assert(kAlloc <= 232448, "beyond the 227 KB of shared memory a CTA may use");
};

// Per-role state shared by the two tile kernels.
struct BwdBars {
    uint64_t* fixed_full;
    uint64_t* ring_full;    // [kStages0]: ring 0 (K or Q) loaded
    uint64_t* ring_empty;   // [kStages0]
    uint64_t* ring1_full;   // [2]: ring 1 (V, or dout and its step's lse / Delta) loaded
    uint64_t* ring1_empty;  // [2]
    uint64_t* s_full;
    uint64_t* p_ready;
    uint64_t* acc_done;
    uint64_t* dp_full;   // dK/dV kernel: dP^T ready (S^T has its own s_full)
    uint64_t* ds_ready;  // dK/dV kernel: dS^T stored
    uint64_t* p_read;    // dK/dV kernel: the element-wise warps have loaded P^T (S^T may be overwritten)
    uint64_t* fixed_empty;  // the item's last products that read the resident tiles are done
    uint64_t* acc_free;     // the element-wise warps have read the item's accumulators out
    uint64_t* item_full;    // [2]
    uint64_t* item_empty;   // [2]
    uint32_t* tmem_slot;
    volatile int* abort_flag;
    BwdItem* items;         // [2]
};

template <int D, bool kDq>
__device__ __forceinline__ BwdBars bwd_setup(uint8_t* smem, int warp) {
    using L = BwdSmem<D, kDq>;
    BwdBars r;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    r.fixed_full = bars;
    r.ring_full = bars + 1;
    r.ring_empty = bars + 4;
    r.s_full = bars + 7;
    r.p_ready = bars + 8;
    r.acc_done = bars + 9;
    r.dp_full = bars + 10;
    r.ds_ready = bars + 11;
    r.p_read = bars + 12;
    r.fixed_empty = bars + 13;
    r.acc_free = bars + 14;
    r.item_full = bars + 15;
    r.item_empty = bars + 17;
    r.ring1_full = bars + 19;
    r.ring1_empty = bars + 21;
    r.tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    r.abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    r.items = reinterpret_cast<BwdItem*>(smem + L::kItems);
    if (threadIdx.x == 0) {
        mbar_init(r.fixed_full, 2);  // two tile loads
        for (int s = 0; s < L::kStages0; ++s) {
            mbar_init(&r.ring_full[s], 1);  // one tile: K (dQ) or Q (dK/dV)
            mbar_init(&r.ring_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&r.ring1_full[s], 1);
            mbar_init(&r.ring1_empty[s], 1);
        }
        mbar_init(r.s_full, 1);
        mbar_init(r.p_ready, kBwdEwWarps);
        mbar_init(r.acc_done, 1);
        mbar_init(r.dp_full, 1);
        mbar_init(r.ds_ready, kBwdEwWarps);
        mbar_init(r.p_read, kBwdEwWarps);
        mbar_init(r.fixed_empty, 1);
        mbar_init(r.acc_free, kBwdEwWarps);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&r.item_full[s], 1);
            mbar_init(&r.item_empty[s], 1 + kBwdEwWarps);  // the MMA lane and the element-wise warps
        }
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

// kCols columns of this thread's row (its TMEM lane) of an f32 accumulator
// at tensor-memory address `taddr`, scaled by `mul`, as bf16 to
// dst + row * row_pitch (nothing is stored when !valid; the loads still run,
// they are warp-wide).
template <int kCols>
__device__ __forceinline__ void bwd_store_rows(uint32_t taddr, float mul, uint8_t* dst,
                                               long long row_pitch, int row, bool valid) {
#pragma unroll
    for (int c = 0; c < kCols / 32; ++c) {
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
// dK, dV: items (key tile kt, KV head hk, sequence b) from the list of key
// tiles, longest first.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ BwdMaps maps, const BwdParams p) {
    using L = BwdSmem<D, false>;
    using T = PrefillSmem<D, ElemBf16>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    if constexpr (L::kNeedsAlignedBase) {
        if (smem != smem_raw) {  // uniform across the CTA: every thread leaves here
            if (threadIdx.x == 0) atomicOr(&g_va_status, kStatusSmemAlign);
            return;
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.H / p.H_kv;
    const long long kv_pitch = static_cast<long long>(p.H_kv) * D * 2;
    const BwdBars bar = bwd_setup<D, false>(smem, warp);
    const uint32_t tmem = *bar.tmem_slot;
    unsigned* status = &g_va_status;
    float* lse_s = reinterpret_cast<float*>(smem + L::kRows);            // [2][128]
    float* dlt_s = reinterpret_cast<float*>(smem + L::kRows + 1024);     // [2][128]
    constexpr uint32_t kS = 0, kDP = 128, kDV = 256, kDK = 256 + D;      // tensor-memory columns
    const int n_items = min(max(p.hdr_k->n_tiles, 0), p.cap_k) * p.H_kv;
    // An item's query rows that see one of its keys ([r0, r1], key_tile_rows)
    // come in n_qt 128-row tiles from qt0; its steps are the G query heads x
    // those tiles.
    auto item_rows = [&](const BwdItem& it, int& qt0, int& n_qt) {
        const int L_q = p.cu_q[it.b + 1] - p.cu_q[it.b], L_k = p.cu_k[it.b + 1] - p.cu_k[it.b];
        int r0, r1;
        key_tile_rows(it.tile, L_q, L_k, p.causal != 0, p.window, r0, r1);
        qt0 = r0 / kBlockM;
        n_qt = it.a1;
    };

    if (warp == kBwdLoadWarp) {
        // ------------------------------------------------------------ producer
        const int T_q = p.cu_q[p.batch], T_k = p.cu_k[p.batch];
        const int q_stride = p.H * D * 2, kv_stride = p.H_kv * D * 2;
        uint32_t ring_n = 0, fixed_n = 0, item_n = 0, issued_q[3] = {0, 0, 0}, issued_d[2] = {0, 0};
        bool ok = true;
        for (;;) {
            int idx = -1;
            if (lane == 0) {
                const int t = atomicAdd(&p.hdr_k->next_item, 1);
                idx = t < n_items ? t : -1;
            }
            idx = __shfl_sync(0xffffffffu, idx, 0);
            BwdItem it{idx, 0, 0, 0, 0, 0, {0, 0}};
            if (idx >= 0) {
                const TileEntry e = p.list_k[idx / p.H_kv];
                it = BwdItem{idx, e.b, e.qt, e.kt_lo, e.kt_hi, idx % p.H_kv, {0, 0}};
            }
            const int slot = item_n & 1;
            if (!(ok = mbar_wait_warp(&bar.item_empty[slot], ((item_n >> 1) & 1) ^ 1, bar.abort_flag, status)))
                break;
            if (lane == 0) {
                bar.items[slot] = it;
                mbar_arrive(&bar.item_full[slot]);
            }
            __syncwarp();
            ++item_n;
            if (idx < 0) break;
            int qt0, n_qt;
            item_rows(it, qt0, n_qt);
            const int n_steps = G * n_qt;
            if (n_steps == 0) continue;
            const int cq = p.cu_q[it.b], ck = p.cu_k[it.b];
            const int L_q = p.cu_q[it.b + 1] - cq;
            const int hk = it.head, k0 = it.tile * kBlockN;
            // K and V once the previous item's last products that read them are done
            if (!(ok = mbar_wait_warp(bar.fixed_empty, (fixed_n & 1) ^ 1, bar.abort_flag, status))) break;
            load_tile<D, ElemBf16>(smem + L::kFixed0, &maps.k, &maps.k8, p.k, ck + k0, T_k, kv_stride,
                                   hk * D, bar.fixed_full, lane);
            load_tile<D, ElemBf16>(smem + L::kFixed1, &maps.v, &maps.v8, p.v, ck + k0, T_k, kv_stride,
                                   hk * D, bar.fixed_full, lane);
            ++fixed_n;
            for (int n = 0; n < n_steps; ++n, ++ring_n) {
                // Q into stage ring_n % 3 of ring 0; dout and the step's lse / Delta
                // rows into stage ring_n % 2 of ring 1
                const int sq = static_cast<int>(ring_n % L::kStages0), sd = ring_n & 1;
                const int h = hk * G + n / n_qt, qt = qt0 + n % n_qt;
                // the tile's 128 rows of {lse * log2(e), Delta} (written by the dQ
                // kernel), four loads per lane in flight while the stages drain
                // (rows past the sequence are masked: any finite value)
                const float2* src = p.rowinfo + h * p.rows_cap + cq + qt * kBlockM;
                float2 ri[kBlockM / 32];
#pragma unroll
                for (int u = 0; u < kBlockM / 32; ++u) {
                    const int r = lane + 32 * u;
                    ri[u] = qt * kBlockM + r < L_q ? src[r] : make_float2(0.f, 0.f);
                }
                if (!(ok = mbar_wait_warp(&bar.ring_empty[sq], ((ring_n / L::kStages0) & 1) ^ 1, bar.abort_flag,
                                          status)))
                    break;
                load_tile<D, ElemBf16>(smem + L::kRing0 + sq * L::kTile, &maps.q, &maps.q8, p.q,
                                       cq + qt * kBlockM, T_q, q_stride, h * D, &bar.ring_full[sq], lane);
                ++issued_q[sq];
                if (!(ok = mbar_wait_warp(&bar.ring1_empty[sd], ((ring_n >> 1) & 1) ^ 1, bar.abort_flag, status)))
                    break;
                // staged negated (the element-wise warps add them); released with
                // the dout tile's arrival on ring1_full
#pragma unroll
                for (int u = 0; u < kBlockM / 32; ++u) {
                    lse_s[sd * kBlockM + lane + 32 * u] = -ri[u].x;
                    dlt_s[sd * kBlockM + lane + 32 * u] = -ri[u].y;
                }
                __syncwarp();
                load_tile<D, ElemBf16>(smem + L::kRing1 + sd * L::kTile, &maps.dout, &maps.dout8, p.dout,
                                       cq + qt * kBlockM, T_q, q_stride, h * D, &bar.ring1_full[sd], lane);
                ++issued_d[sd];
            }
            if (!ok) break;
        }
        if (!ok && lane == 0) {
            const unsigned long long t0 = global_timer_ns();
            bwd_drain(bar.fixed_full, fixed_n, t0);
            for (int sq = 0; sq < L::kStages0; ++sq) bwd_drain(&bar.ring_full[sq], issued_q[sq], t0);
            bwd_drain(&bar.ring1_full[0], issued_d[0], t0);
            bwd_drain(&bar.ring1_full[1], issued_d[1], t0);
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
            // S^T = K Q^T for step m (Q of ring-0 stage m % 3, K-major operands, K = D)
            auto issue_s = [&](uint32_t m) {
                const uint32_t ring = ((m % L::kStages0) * L::kTile) >> 4;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * T::kChunkBytes + (kk & 3) * 32) >> 4;
                    mma_ss_lh<idesc_ss>(tmem + kS, static_cast<uint32_t>(dk_) + off, hi_k,
                                        static_cast<uint32_t>(dq_k) + ring + off, hi_k, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar.s_full);
            };
            // dP^T = V dout^T for step m (dout of ring-1 stage m & 1, K-major operands, K = D)
            auto issue_dp = [&](uint32_t m) {
                const uint32_t ring = ((m & 1) * L::kTile) >> 4;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * T::kChunkBytes + (kk & 3) * 32) >> 4;
                    mma_ss_lh<idesc_ss>(tmem + kDP, static_cast<uint32_t>(dv_) + off, hi_k,
                                        static_cast<uint32_t>(dd_k) + ring + off, hi_k, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar.dp_full);
            };
            uint32_t g = 0, fixed_n = 0, acc_n = 0, item_n = 0;
            bool ok = true;
            for (;;) {
                const int slot = item_n & 1;
                if (!(ok = mbar_wait(&bar.item_full[slot], (item_n >> 1) & 1, bar.abort_flag, status))) break;
                const BwdItem it = bar.items[slot];
                mbar_arrive(&bar.item_empty[slot]);
                ++item_n;
                if (it.idx < 0) break;
                const int n_steps = G * it.a1;
                if (n_steps == 0) continue;
                if (!(ok = mbar_wait(bar.fixed_full, fixed_n & 1, bar.abort_flag, status))) break;
                ++fixed_n;
                if (!(ok = mbar_wait(&bar.ring_full[g % L::kStages0], (g / L::kStages0) & 1, bar.abort_flag,
                                     status)))
                    break;
                tc_fence_after();
                issue_s(g);
                if (!(ok = mbar_wait(&bar.ring1_full[g & 1], (g >> 1) & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                issue_dp(g);
                // the item's last products that read K and V (its last S^T and dP^T)
                // are issued: the next item's K and V may load while the rest runs
                if (n_steps == 1) mma_commit(bar.fixed_empty);
                // Order per step m: S^T(m+1) as soon as the element-wise warps have
                // loaded S^T(m) (P^T and dS^T go to the dP^T columns, so the S^T
                // columns are free and the next S^T runs while P^T(m) is formed), then
                // dV(m) and dK(m) once P^T(m) and dS^T(m) are stored, then dP^T(m+1),
                // which overwrites them.
                for (int n = 0; n < n_steps && ok; ++n) {
                    const uint32_t m = g + n;
                    const int sq = static_cast<int>(m % L::kStages0), sd = m & 1;
                    const uint32_t ring_q = (sq * L::kTile) >> 4, ring_d = (sd * L::kTile) >> 4;
                    if (n + 1 < n_steps) {
                        if (!(ok = mbar_wait(&bar.ring_full[(m + 1) % L::kStages0], ((m + 1) / L::kStages0) & 1,
                                             bar.abort_flag, status)))
                            break;
                        if (!(ok = mbar_wait(bar.p_read, m & 1, bar.abort_flag, status))) break;
                        tc_fence_after();
                        issue_s(m + 1);
                    }
                    if (!(ok = mbar_wait(bar.ds_ready, m & 1, bar.abort_flag, status))) break;
                    // the first dV of an item overwrites the accumulators: the previous
                    // item's must have been read out
                    if (n == 0 && acc_n > 0 &&
                        !(ok = mbar_wait(bar.acc_free, (acc_n - 1) & 1, bar.abort_flag, status)))
                        break;
                    tc_fence_after();
                    // dV += P^T dout and dK += dS^T Q (A from tensor memory: P^T at
                    // kDP + bwd_kcol, dS^T 32 columns on; B MN-major, K = 128 query rows)
#pragma unroll
                    for (int kk = 0; kk < kBlockM / 16; ++kk)
                        mma_ts_lh<idesc_ts>(tmem + kDV, tmem + kDP + bwd_kcol(kk),
                                            static_cast<uint32_t>(dd_mn) + ring_d + ((kk * 16 * 128) >> 4), hi_mn,
                                            (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < kBlockM / 16; ++kk)
                        mma_ts_lh<idesc_ts>(tmem + kDK, tmem + kDP + 32 + bwd_kcol(kk),
                                            static_cast<uint32_t>(dq_mn) + ring_q + ((kk * 16 * 128) >> 4), hi_mn,
                                            (n > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&bar.ring_empty[sq]);
                    mma_commit(&bar.ring1_empty[sd]);
                    if (n + 1 < n_steps) {
                        if (!(ok = mbar_wait(&bar.ring1_full[(m + 1) & 1], ((m + 1) >> 1) & 1, bar.abort_flag,
                                             status)))
                            break;
                        tc_fence_after();
                        issue_dp(m + 1);
                        if (n + 2 == n_steps) mma_commit(bar.fixed_empty);
                    }
                }
                if (!ok) break;
                mma_commit(bar.acc_done);
                g += n_steps;
                ++acc_n;
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ element-wise
        const int quarter = warp & 3;                       // TMEM lane quarter
        const int ch = warp >> 2;                           // query columns 64 ch .. 64 ch + 63
        const int jj = quarter * 32 + lane;                 // key row of the tile (TMEM lane)
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
        uint32_t g = 0, acc_n = 0, item_n = 0;
        bool ok = true;
        for (;;) {
            const int slot = item_n & 1;
            if (!(ok = mbar_wait_warp(&bar.item_full[slot], (item_n >> 1) & 1, bar.abort_flag, status))) break;
            const BwdItem it = bar.items[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.item_empty[slot]);
            ++item_n;
            if (it.idx < 0) break;
            const int hk = it.head;
            const int cq = p.cu_q[it.b], ck = p.cu_k[it.b];
            const int L_q = p.cu_q[it.b + 1] - cq, L_k = p.cu_k[it.b + 1] - ck;
            const int k0 = it.tile * kBlockN;
            const int delta_k = L_k - L_q;
            const int j = k0 + jj;                          // key index in the sequence
            int qt0, n_qt;
            item_rows(it, qt0, n_qt);
            const int n_steps = G * n_qt;
            if (n_steps == 0) {
                // no query sees these keys: their gradients are zero (this warp's
                // half of the columns of its rows)
                if (j < L_k) {
                    const long long off = (static_cast<long long>(ck) + j) * kv_pitch + hk * D * 2 + ch * D;
#pragma unroll
                    for (int c = 0; c < D / 16; ++c) {
                        reinterpret_cast<uint4*>(p.dk + off)[c] = make_uint4(0u, 0u, 0u, 0u);
                        reinterpret_cast<uint4*>(p.dv + off)[c] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                continue;
            }
            // query rows that see key j: [i_lo, i_hi] (empty when j is past the keys)
            int i_lo = 0, i_hi = L_q - 1;
            if (p.causal || p.window > 0) i_lo = max(0, j - delta_k);
            if (p.window > 0) i_hi = min(i_hi, j - delta_k + p.window - 1);
            if (j >= L_k) i_hi = -1;
            const unsigned i_span = i_hi >= i_lo ? static_cast<unsigned>(i_hi - i_lo) : 0u;
            const int i_base = i_hi >= i_lo ? i_lo : (1 << 30);
            for (int n = 0; n < n_steps; ++n) {
                const uint32_t m = g + n;  // step count across items
                const int st = m & 1;
                const int qt = qt0 + n % n_qt;
                if (!(ok = mbar_wait_warp(bar.s_full, m & 1, bar.abort_flag, status))) break;
                // the producer's stores of this step's logsumexp and Delta rows are
                // released by its arrival with the dout tile on ring1_full
                if (!(ok = mbar_wait_warp(&bar.ring1_full[st], (m >> 1) & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                const float* nl2 = lse_s + st * kBlockM;  // -lse * log2(e) per query column
                const float* ndl = dlt_s + st * kBlockM;  // -Delta per query column
                // every pair of this warp's keys and query columns visible?  Then the
                // loops below skip the mask (every tile of a non-causal sequence but
                // its ragged last one)
                const int i0 = qt * kBlockM + ch * 64;
                const bool full = __all_sync(0xffffffffu, i_span != 0u && i_base <= i0 &&
                                                              i0 + 63 <= i_base + static_cast<int>(i_span));
                // P^T = exp2(s * log2(e) / sqrt(D) - lse * log2(e)) on visible pairs, as
                // bf16 pairs kept in registers until dP^T has been read
                uint32_t pk[2][16];
                {
                    uint32_t sbuf[2][32];
                    tmem_ld32(tmem + lane_addr + kS + ch * 64, sbuf[0]);
                    tmem_ld32(tmem + lane_addr + kS + ch * 64 + 32, sbuf[1]);
                    tmem_wait_ld();
                    // every S^T value of this warp is in registers: the next S^T may land
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar.p_read);
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = 2 * ch + cc;
                        const uint32_t* sr = sbuf[cc];
                        // scale and shift as packed pairs, then the mask (only on tiles
                        // where some pair of this warp is not visible)
                        float pv[32];
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 nl = *reinterpret_cast<const float4*>(nl2 + c * 32 + e);
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), scale2,
                                             f2_pack(nl.x, nl.y)),
                                      pv[e], pv[e + 1]);
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3])), scale2,
                                             f2_pack(nl.z, nl.w)),
                                      pv[e + 2], pv[e + 3]);
                        }
#pragma unroll
                        for (int e = 0; e < 32; ++e) pv[e] = ex2_approx(pv[e]);
                        if (!full) {
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const int i = qt * kBlockM + c * 32 + e;
                                pv[e] = static_cast<unsigned>(i - i_base) <= i_span ? pv[e] : 0.f;
                            }
                        }
#pragma unroll
                        for (int e = 0; e < 32; e += 2) pk[cc][e / 2] = pack_bf16x2(pv[e], pv[e + 1]);
                    }
                }
                // dS^T = P^T (dP^T - Delta) from the bf16 P^T; then P^T at kDP +
                // bwd_pcol(c) and dS^T 32 columns on, over dP^T columns this warp has
                // read
                if (!(ok = mbar_wait_warp(bar.dp_full, m & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                {
                    uint32_t dbuf[2][32];
                    tmem_ld32(tmem + lane_addr + kDP + ch * 64, dbuf[0]);
                    tmem_ld32(tmem + lane_addr + kDP + ch * 64 + 32, dbuf[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = 2 * ch + cc;
                        const uint32_t* dr = dbuf[cc];
                        const uint32_t* pr = pk[cc];
                        // dS = P (dP - Delta) on packed pairs; a masked pair has P = 0 and a
                        // finite dP - Delta (rows past the sequence stage Delta = 0), so it
                        // stays 0
                        uint32_t dk16[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 nd = *reinterpret_cast<const float4*>(ndl + c * 32 + e);
                            float ds[4];
#pragma unroll
                            for (int u = 0; u < 4; u += 2) {
                                const uint32_t w = pr[(e + u) / 2];
                                const uint64_t p2 = f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
                                const uint64_t d2 = f2_add(f2_pack(__uint_as_float(dr[e + u]), __uint_as_float(dr[e + u + 1])),
                                                           u == 0 ? f2_pack(nd.x, nd.y) : f2_pack(nd.z, nd.w));
                                f2_unpack(f2_mul(p2, d2), ds[u], ds[u + 1]);
                            }
                            dk16[e / 2] = pack_bf16x2(ds[0], ds[1]);
                            dk16[e / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
                        }
                        tmem_st16(tmem + lane_addr + kDP + bwd_pcol(c), pk[cc]);
                        tmem_st16(tmem + lane_addr + kDP + bwd_pcol(c) + 32, dk16);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar.ds_ready);
            }
            if (!ok) break;
            if (!(ok = mbar_wait_warp(bar.acc_done, acc_n & 1, bar.abort_flag, status))) break;
            tc_fence_after();
            // this warp's half of the D columns of its 32 key rows
            const bool valid = j < L_k;
            const long long col = hk * D * 2 + ch * D;  // bytes
            uint8_t* base_v = p.dv + (static_cast<long long>(ck) + k0) * kv_pitch + col;
            uint8_t* base_k = p.dk + (static_cast<long long>(ck) + k0) * kv_pitch + col;
            bwd_store_rows<D / 2>(tmem + lane_addr + kDV + ch * (D / 2), 1.f, base_v, kv_pitch, jj, valid);
            bwd_store_rows<D / 2>(tmem + lane_addr + kDK + ch * (D / 2), p.scale, base_k, kv_pitch, jj, valid);
            // the accumulators are in registers: the next item's first dV may overwrite them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.acc_free);
            g += n_steps;
            ++acc_n;
        }
    }
    bwd_teardown<D>(bar, tmem, warp);
}

// ---------------------------------------------------------------------------
// dQ: items (query tile qt, query head h, sequence b) from the list of query
// tiles, longest first.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dq_kernel(const __grid_constant__ BwdMaps maps, const BwdParams p) {
    using L = BwdSmem<D, true>;
    using T = PrefillSmem<D, ElemBf16>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    if constexpr (L::kNeedsAlignedBase) {
        if (smem != smem_raw) {  // uniform across the CTA: every thread leaves here
            if (threadIdx.x == 0) atomicOr(&g_va_status, kStatusSmemAlign);
            return;
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const BwdBars bar = bwd_setup<D, true>(smem, warp);
    const uint32_t tmem = *bar.tmem_slot;
    unsigned* status = &g_va_status;
    constexpr uint32_t kS = 0, kDP = 128, kDQ = 256;  // tensor-memory columns
    const long long q_pitch = static_cast<long long>(p.H) * D * 2;
    const int n_items = min(max(p.hdr_q->n_tiles, 0), p.cap_q) * p.H;
    const int G = p.H / p.H_kv;

    if (warp == kBwdLoadWarp) {
        // ------------------------------------------------------------ producer
        const int T_q = p.cu_q[p.batch], T_k = p.cu_k[p.batch];
        const int q_stride = p.H * D * 2, kv_stride = p.H_kv * D * 2;
        uint32_t ring_n = 0, fixed_n = 0, item_n = 0, issued_k[3] = {0, 0, 0}, issued_v[2] = {0, 0};
        bool ok = true;
        for (;;) {
            // claim the next item (longest first across the grid) and publish it
            int idx = -1;
            if (lane == 0) {
                const int t = atomicAdd(&p.hdr_q->next_item, 1);
                idx = t < n_items ? t : -1;
            }
            idx = __shfl_sync(0xffffffffu, idx, 0);
            BwdItem it{idx, 0, 0, 0, 0, 0, {0, 0}};
            if (idx >= 0) {
                const TileEntry e = p.list_q[idx / p.H];
                it = BwdItem{idx, e.b, e.qt, e.kt_lo, e.kt_hi, idx % p.H, {0, 0}};
            }
            const int slot = item_n & 1;
            if (!(ok = mbar_wait_warp(&bar.item_empty[slot], ((item_n >> 1) & 1) ^ 1, bar.abort_flag, status)))
                break;
            if (lane == 0) {
                bar.items[slot] = it;
                mbar_arrive(&bar.item_full[slot]);
            }
            __syncwarp();
            ++item_n;
            if (idx < 0) break;
            const int n_steps = it.a1 - it.a0;
            if (n_steps <= 0) continue;
            const int cq = p.cu_q[it.b], ck = p.cu_k[it.b];
            const int h = it.head, hk = h / G, q0 = it.tile * kBlockM;
            // Q and dout once the previous item's last products that read them are done
            if (!(ok = mbar_wait_warp(bar.fixed_empty, (fixed_n & 1) ^ 1, bar.abort_flag, status))) break;
            load_tile<D, ElemBf16>(smem + L::kFixed0, &maps.q, &maps.q8, p.q, cq + q0, T_q, q_stride, h * D,
                                   bar.fixed_full, lane);
            load_tile<D, ElemBf16>(smem + L::kFixed1, &maps.dout, &maps.dout8, p.dout, cq + q0, T_q, q_stride,
                                   h * D, bar.fixed_full, lane);
            ++fixed_n;
            for (int n = 0; n < n_steps; ++n, ++ring_n) {
                // K into stage ring_n % 3 of ring 0, V into stage ring_n % 2 of ring 1
                const int sk = static_cast<int>(ring_n % L::kStages0), sv = ring_n & 1, kt = it.a0 + n;
                if (!(ok = mbar_wait_warp(&bar.ring_empty[sk], ((ring_n / L::kStages0) & 1) ^ 1, bar.abort_flag,
                                          status)))
                    break;
                load_tile<D, ElemBf16>(smem + L::kRing0 + sk * L::kTile, &maps.k, &maps.k8, p.k,
                                       ck + kt * kBlockN, T_k, kv_stride, hk * D, &bar.ring_full[sk], lane);
                ++issued_k[sk];
                if (!(ok = mbar_wait_warp(&bar.ring1_empty[sv], ((ring_n >> 1) & 1) ^ 1, bar.abort_flag, status)))
                    break;
                load_tile<D, ElemBf16>(smem + L::kRing1 + sv * L::kTile, &maps.v, &maps.v8, p.v,
                                       ck + kt * kBlockN, T_k, kv_stride, hk * D, &bar.ring1_full[sv], lane);
                ++issued_v[sv];
            }
            if (!ok) break;
        }
        if (!ok && lane == 0) {
            const unsigned long long t0 = global_timer_ns();
            bwd_drain(bar.fixed_full, fixed_n, t0);
            for (int sk = 0; sk < L::kStages0; ++sk) bwd_drain(&bar.ring_full[sk], issued_k[sk], t0);
            bwd_drain(&bar.ring1_full[0], issued_v[0], t0);
            bwd_drain(&bar.ring1_full[1], issued_v[1], t0);
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
            // S = Q K^T for step m (K of ring-0 stage m % 3, K-major operands, K = D)
            auto issue_s = [&](uint32_t m) {
                const uint32_t ring = ((m % L::kStages0) * L::kTile) >> 4;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * T::kChunkBytes + (kk & 3) * 32) >> 4;
                    mma_ss_lh<idesc_ss>(tmem + kS, static_cast<uint32_t>(dq_) + off, hi_k,
                                        static_cast<uint32_t>(dk_k) + ring + off, hi_k, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar.s_full);
            };
            uint32_t g = 0, fixed_n = 0, acc_n = 0, item_n = 0;
            bool ok = true;
            for (;;) {
                const int slot = item_n & 1;
                if (!(ok = mbar_wait(&bar.item_full[slot], (item_n >> 1) & 1, bar.abort_flag, status))) break;
                const BwdItem it = bar.items[slot];
                mbar_arrive(&bar.item_empty[slot]);
                ++item_n;
                if (it.idx < 0) break;
                const int n_steps = it.a1 - it.a0;
                if (n_steps <= 0) continue;
                if (!(ok = mbar_wait(bar.fixed_full, fixed_n & 1, bar.abort_flag, status))) break;
                ++fixed_n;
                if (!(ok = mbar_wait(&bar.ring_full[g % L::kStages0], (g / L::kStages0) & 1, bar.abort_flag,
                                     status)))
                    break;
                tc_fence_after();
                issue_s(g);
                // Order per step m: dP(m), S(m+1) once the element-wise warps have read
                // S(m), dQ(m) once dS(m) is stored.  The next S so runs while dS is
                // formed; dP(m+1) overwrites dS(m) and follows dQ(m).  V(m) is
                // released as soon as dP(m) completes, K(m) once dQ(m) does.
                for (int n = 0; n < n_steps && ok; ++n) {
                    const uint32_t m = g + n;
                    const int sk = static_cast<int>(m % L::kStages0), sv = m & 1;
                    const uint32_t ring_k = (sk * L::kTile) >> 4, ring_v = (sv * L::kTile) >> 4;
                    if (!(ok = mbar_wait(&bar.ring1_full[sv], (m >> 1) & 1, bar.abort_flag, status))) break;
                    tc_fence_after();
                    // dP = dout V^T (K-major operands, K = D)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * T::kChunkBytes + (kk & 3) * 32) >> 4;
                        mma_ss_lh<idesc_ss>(tmem + kDP, static_cast<uint32_t>(dd_) + off, hi_k,
                                            static_cast<uint32_t>(dv_k) + ring_v + off, hi_k, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar.dp_full);
                    mma_commit(&bar.ring1_empty[sv]);
                    // the item's last products that read Q and dout (its last S and dP)
                    // are issued: the next item's Q and dout may load while dQ runs
                    if (n + 1 == n_steps) mma_commit(bar.fixed_empty);
                    if (n + 1 < n_steps) {
                        if (!(ok = mbar_wait(&bar.ring_full[(m + 1) % L::kStages0], ((m + 1) / L::kStages0) & 1,
                                             bar.abort_flag, status)))
                            break;
                        if (!(ok = mbar_wait(bar.p_read, m & 1, bar.abort_flag, status))) break;
                        tc_fence_after();
                        issue_s(m + 1);
                    }
                    if (!(ok = mbar_wait(bar.p_ready, m & 1, bar.abort_flag, status))) break;
                    // the first dQ of an item overwrites the accumulator: the previous
                    // item's must have been read out
                    if (n == 0 && acc_n > 0 &&
                        !(ok = mbar_wait(bar.acc_free, (acc_n - 1) & 1, bar.abort_flag, status)))
                        break;
                    tc_fence_after();
                    // dQ += dS K (A from tensor memory, B = K MN-major, K = 128 keys)
#pragma unroll
                    for (int kk = 0; kk < kBlockN / 16; ++kk) {
                        mma_ts_lh<idesc_ts>(tmem + kDQ, tmem + kDP + bwd_kcol(kk),
                                            static_cast<uint32_t>(dk_mn) + ring_k + ((kk * 16 * 128) >> 4), hi_mn,
                                            (n > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&bar.ring_empty[sk]);
                }
                if (!ok) break;
                mma_commit(bar.acc_done);
                g += n_steps;
                ++acc_n;
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ element-wise
        const int quarter = warp & 3;        // TMEM lane quarter
        const int ch = warp >> 2;            // key columns 64 ch .. 64 ch + 63
        const int ii = quarter * 32 + lane;  // query row of the tile (TMEM lane)
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t g = 0, acc_n = 0, item_n = 0;
        bool ok = true;
        for (;;) {
            const int slot = item_n & 1;
            if (!(ok = mbar_wait_warp(&bar.item_full[slot], (item_n >> 1) & 1, bar.abort_flag, status))) break;
            const BwdItem it = bar.items[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.item_empty[slot]);
            ++item_n;
            if (it.idx < 0) break;
            const int h = it.head;
            const int cq = p.cu_q[it.b], ck = p.cu_k[it.b];
            const int L_q = p.cu_q[it.b + 1] - cq, L_k = p.cu_k[it.b + 1] - ck;
            const int q0 = it.tile * kBlockM;
            const int i = q0 + ii;
            const bool row_valid = i < L_q;
            const int n_steps = it.a1 - it.a0;
            if (n_steps <= 0) {
                // these rows see no key: dq is zero (this warp's half of the columns)
                if (row_valid) {
                    uint4* o = reinterpret_cast<uint4*>(p.dq + (static_cast<long long>(cq) + i) * q_pitch +
                                                        h * D * 2 + ch * D);
#pragma unroll
                    for (int c = 0; c < D / 16; ++c) o[c] = make_uint4(0u, 0u, 0u, 0u);
                }
                continue;
            }
            float l2 = 0.f, dl = 0.f;
            int lo = 0, hi = -1;
            if (row_valid) {
                const size_t row = static_cast<size_t>(cq + i) * p.H + h;
                const float l = p.lse[row];
                l2 = l == -INFINITY ? 0.f : l * 1.4426950408889634f;
                // Delta_i = dout_i . out_i, kept here and stored for the dK/dV kernel
                const uint4* o4 = reinterpret_cast<const uint4*>(p.out + row * (D * 2));
                const uint4* g4 = reinterpret_cast<const uint4*>(p.dout + row * (D * 2));
                float acc = 0.f;
#pragma unroll 4
                for (int c = 0; c < D / 8; ++c) {
                    const uint4 a = o4[c], gg = g4[c];
                    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc = fmaf(__uint_as_float(av[e] << 16), __uint_as_float(gv[e] << 16), acc);
                        acc = fmaf(__uint_as_float(av[e] & 0xFFFF0000u), __uint_as_float(gv[e] & 0xFFFF0000u), acc);
                    }
                }
                dl = acc;
                if (ch == 0) p.rowinfo[h * p.rows_cap + cq + i] = make_float2(l2, acc);
                row_key_interval(i, L_q, L_k, p.causal != 0, p.window, lo, hi);
            }
            const unsigned span = hi >= lo ? static_cast<unsigned>(hi - lo) : 0u;
            const int base = hi >= lo ? lo : (1 << 30);
            const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
            const uint64_t nl2 = f2_pack(-l2, -l2), ndl2 = f2_pack(-dl, -dl);
            for (int n = 0; n < n_steps; ++n) {
                const int kt = it.a0 + n;
                const uint32_t m = g + n;  // step count across items
                if (!(ok = mbar_wait_warp(bar.s_full, m & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                // all of this warp's rows see every key of its columns?  (skip the mask)
                const int k0c = kt * kBlockN + ch * 64;
                const bool full = __all_sync(0xffffffffu, hi >= lo && lo <= k0c && k0c + 63 <= hi);
                // P = exp2(s * log2(e) / sqrt(D) - lse * log2(e)) on visible pairs, in
                // registers; then S may be overwritten by the next step's product
                float pv[64];
                {
                    uint32_t sbuf[2][32];
                    tmem_ld32(tmem + lane_addr + kS + ch * 64, sbuf[0]);
                    tmem_ld32(tmem + lane_addr + kS + ch * 64 + 32, sbuf[1]);
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar.p_read);
#pragma unroll
                    for (int e = 0; e < 64; e += 2)
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(sbuf[e >> 5][e & 31]),
                                                 __uint_as_float(sbuf[e >> 5][(e & 31) + 1])),
                                         scale2, nl2),
                                  pv[e], pv[e + 1]);
#pragma unroll
                    for (int e = 0; e < 64; ++e) pv[e] = ex2_approx(pv[e]);
                    if (!full) {
#pragma unroll
                        for (int e = 0; e < 64; ++e)
                            pv[e] = static_cast<unsigned>(k0c + e - base) <= span ? pv[e] : 0.f;
                    }
                }
                // dS = P (dP - Delta) as bf16 at kDP + bwd_pcol(c), over dP columns read
                if (!(ok = mbar_wait_warp(bar.dp_full, m & 1, bar.abort_flag, status))) break;
                tc_fence_after();
                {
                    uint32_t dbuf[2][32];
                    tmem_ld32(tmem + lane_addr + kDP + ch * 64, dbuf[0]);
                    tmem_ld32(tmem + lane_addr + kDP + ch * 64 + 32, dbuf[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t dk16[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            // a masked pair has P = 0 and a finite dP - Delta: it stays 0
                            float d0, d1;
                            f2_unpack(f2_mul(f2_pack(pv[cc * 32 + e], pv[cc * 32 + e + 1]),
                                             f2_add(f2_pack(__uint_as_float(dbuf[cc][e]), __uint_as_float(dbuf[cc][e + 1])),
                                                    ndl2)),
                                      d0, d1);
                            dk16[e / 2] = pack_bf16x2(d0, d1);
                        }
                        tmem_st16(tmem + lane_addr + kDP + bwd_pcol(2 * ch + cc), dk16);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar.p_ready);
            }
            if (!ok) break;
            if (!(ok = mbar_wait_warp(bar.acc_done, acc_n & 1, bar.abort_flag, status))) break;
            tc_fence_after();
            // this warp's half of the D columns of its 32 query rows
            uint8_t* base_q = p.dq + (static_cast<long long>(cq) + q0) * q_pitch + h * D * 2 + ch * D;
            bwd_store_rows<D / 2>(tmem + lane_addr + kDQ + ch * (D / 2), p.scale, base_q, q_pitch, ii,
                                  row_valid);
            // the accumulator is in registers: the next item's first dQ may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.acc_free);
            g += n_steps;
            ++acc_n;
        }
    }
    bwd_teardown<D>(bar, tmem, warp);
}

}  // namespace va
