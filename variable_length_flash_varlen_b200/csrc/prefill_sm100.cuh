// Persistent, warp-specialised packed-attention forward for sm_100a.
//
// A work item is one 256-row query block of one (sequence, query head),
// split into two 128-row MMA tiles ("halves") that share every K/V tile of
// 128 keys.  Per CTA (320 threads, one CTA per SM):
//   warps 0-3   softmax for half 0, warps 4-7 softmax for half 1: one query
//               row per thread; online softmax in base 2 with a lazily moved
//               reference max, P written back to tensor memory as bf16, O
//               rescaled in place when the reference moves, epilogue O / l
//               and logsumexp
//   warp 8      tensor-memory owner and MMA issuer (one lane):
//               S_h = Q_h K^T (SS form), O_h += P_h V (P_h read from tensor
//               memory), issued as PV_0[j], QK_0[j+1], PV_1[j], QK_1[j+1] so
//               one half's MMAs run while the other half's softmax does
//   warp 9      producer: claims work items from a grid-wide counter (longest
//               first), TMA tile loads of Q, K, V into 128-byte-swizzled
//               shared memory (8-row boxes and one group of plain loads for
//               a tile that runs past the end of the packed tensor)
// Tensor memory (512 columns): S_0 at 0, S_1 at 128 (P_h aliases the first
// 64 columns of S_h, or 32 for E4M3; the residual variant's P - bf16(P) the
// next 64), O_0 at 256, O_1 at 256 + D.
//
// Two element formats share this code (the ElemBf16 / ElemE4m3 traits):
// bf16 inputs and output (kind::f16 MMAs), and E4M3 inputs and output with
// per-tensor scales (kind::f8f6f4 MMAs; the FP8 forward of boostr flash.rs,
// FlashAttentionOps::flash_attention_fwd_fp8), where the Q and K scales are
// folded into the score scale and the V and output scales into the
// epilogue's 1 / l.
//
// The recurrence is the tiled one of realizar 0.8.4 attention.rs, IMP-111
// (online_softmax / tiled_single_head_attention): running max, running sum
// rescaled by exp(old - new), output rescaled alongside, normalised at the end.
// Packed addressing and GQA head mapping follow boostr 0.2.0
// varlen_attention.rs, VarLenAttentionOps docs ("Layout contract", "GQA
// key/value head mapping"): kv_head = q_head / (H / H_kv); K/V are read for
// the head that needs them and never repeated in memory.
#pragma once

#include <cuda_bf16.h>

#include "f32x2.cuh"
#include "ptx.cuh"
#include "schedule.cuh"
#include "status.cuh"

namespace va {

constexpr int kPrefillThreads = 320;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may grow to 2^8 before O is rescaled

// Input element formats.  bf16: Q, K, V and O in bf16, P rounded to bf16 for
// the tensor-core PV product (kind::f16, K = 16 per instruction).  E4M3:
// Q, K, V and O in 8-bit E4M3 with per-tensor scales (boostr flash.rs,
// FlashAttentionOps::flash_attention_fwd_fp8: FP32 accumulation inside), P
// rounded to E4M3 (kind::f8f6f4, K = 32 per instruction).  Either way one
// MMA step consumes 32 bytes of every operand row.
struct ElemBf16 {
    static constexpr int kBytes = 2;
    static constexpr bool kFp8 = false;
};
struct ElemE4m3 {
    static constexpr int kBytes = 1;
    static constexpr bool kFp8 = true;
};

struct PrefillParams {
    const int* cu_q;
    const int* cu_k;
    const int* seqused_k;  // optional key counts of a capacity-strided cache (else NULL)
    int batch, H, H_kv, causal, window;
    const TileEntry* tiles;
    SchedHeader* hdr;
    int tile_capacity;  // entries the list can hold; the count read from hdr is clamped to it
    const uint8_t* q;  // element bytes of the packed tensors (bf16 or E4M3)
    const uint8_t* k;
    const uint8_t* v;
    uint8_t* out;
    float* lse;
    float scale_log2;  // log2(e) / sqrt(D), times q_scale * k_scale for E4M3 inputs
    float out_mul;     // 1 for bf16; v_scale / o_scale for E4M3 (dequantize V, quantize O)
    int after_residual;  // the residual variant was launched between the build and this grid
};

template <int D, class E>
struct PrefillSmem {
    static constexpr int kRowBytes = D * E::kBytes;             // one token row of one head
    static constexpr int kChunks = kRowBytes / 128;             // 128-byte swizzle atoms per row
    static_assert(kChunks >= 1 && kRowBytes % 128 == 0, "rows must be whole 128-byte atoms");
    static constexpr int kChunkCols = 128 / E::kBytes;          // elements per atom row
    static constexpr int kChunkBytes = 128 * 128;               // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    // K/V ring depth (tiles of kBlockN keys): E4M3 tiles are half the size, so
    // the same shared memory holds twice the stages
    static constexpr int kStages = E::kFp8 ? 4 : 2;
    static constexpr int kQ = 0;                    // two Q tiles
    static constexpr int kK = kQ + 2 * kTileBytes;
    static constexpr int kV = kK + kStages * kTileBytes;
    static constexpr int kBar = kV + kStages * kTileBytes;
    // q_full[2], q_empty, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_half[2],
    // p_full[2], o_done[2], item_full[2], item_empty[2]
    static constexpr int kNumBars = 3 + 4 * kStages + 12;
    static constexpr int kMisc = kBar + kNumBars * 8;  // tmem slot, abort flag, item ring[2]
    static constexpr int kItems = kMisc + 16;          // the ring's decoded items [2]
    // epilogue staging, per softmax warp 32 rows x 64 bytes (one 64-byte column block of O)
    static constexpr int kStage = (kItems + 2 * 64 + 15) & ~15;
    static constexpr int kBytes = kStage + 8 * 2048;
    // slack for 1024-byte alignment; never below 120 KB so that at most one CTA
    // (and one 512-column tensor-memory allocation) is resident per SM
    static constexpr int kAlloc = (kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024;
    __host__ __device__ static constexpr uint32_t tmem_s(int x) { return x ? 128u : 0u; }
    __host__ __device__ static constexpr uint32_t tmem_o(int x) { return 256u + x * D; }
};

// Everything every role derives from a work-item index.
struct Item {
    int b, qb, h, hk;
    int L_q, L_k;
    int q_row0, k_row0;   // first packed row of the query block / of the sequence's keys
    int lo, hi;           // key-tile range of the block (union of the halves)
    int lo_h[2], hi_h[2]; // key-tile range of each 128-row half
};
static_assert(sizeof(Item) <= 64, "an item must fit its 64-byte ring slot");

__device__ __forceinline__ void decode_item(const PrefillParams& p, int idx, int group, Item& it) {
    // through L2: the main variant reads the list without a grid-dependency
    // wait on the grid that wrote it (see the kernel's start)
    const int4 te = __ldcg(reinterpret_cast<const int4*>(p.tiles) + idx / p.H);
    static_assert(sizeof(TileEntry) == sizeof(int4), "a list entry is one 16-byte load");
    it.h = idx % p.H;
    it.hk = it.h / group;
    it.b = te.x;
    it.qb = te.y;
    it.lo = te.z;
    it.hi = te.w;
    const int cq = p.cu_q[it.b], ck = p.cu_k[it.b];
    it.L_q = p.cu_q[it.b + 1] - cq;
    it.L_k = seq_key_count(p.cu_k, p.seqused_k, it.b);
    it.q_row0 = cq + it.qb * kBlockQ;
    it.k_row0 = ck;
#pragma unroll
    for (int x = 0; x < 2; ++x)
        rows_key_range(it.qb * kBlockQ + x * kBlockM, kBlockM, it.L_q, it.L_k, p.causal != 0,
                       p.window, it.lo_h[x], it.hi_h[x]);
}

__device__ __forceinline__ bool takes_part(const Item& it, int x, int kt) {
    return it.lo_h[x] <= kt && kt < it.hi_h[x];
}

// Tensor maps of the three inputs, each as a 2-D view [rows][heads * D] with
// 128-byte-wide boxes and 128-byte swizzle: one with 128-row boxes for whole
// tiles and one with 8-row boxes (one swizzle atom high) for a tile that runs
// past the end of the packed tensor.  The row extent of every map is only an
// upper bound of the packed length (batch * max_seqlen; the exact total lives
// in cu_seqlens on the device), so no box may cover a row at or past it.
struct PrefillMaps {
    CUtensorMap q, k, v;     // 128-row boxes
    CUtensorMap q8, k8, v8;  // 8-row boxes
};

// A 128-row tile whose rows run past the packed length `T`, in the
// 128-byte-swizzle layout a full-tile copy would produce, rows >= T zero.
// The whole groups of 8 rows before T come by TMA in 8-row boxes (a box
// written at a 1024-byte-aligned offset carries the same swizzle phase as
// those rows of a full box); the one partial group is read with plain loads,
// all in flight at once, and the rows after it are zero-filled.  Completion is
// signalled on `full` (one arrival, carrying the TMA byte count).
// `src` is the tensor's first byte, `row_stride` its row pitch in bytes and
// `col0` the head's first element column.
template <int D, class E>
__device__ __forceinline__ void load_tile_ragged(uint8_t* dst, const CUtensorMap* map8,
                                                 const uint8_t* src, int row0, int T,
                                                 int row_stride, int col0, uint64_t* full, int lane) {
    using L = PrefillSmem<D, E>;
    constexpr int kVecPerRow = L::kRowBytes / 16;     // 16-byte vectors per row
    constexpr int kTailVec = 8 * kVecPerRow;          // one 8-row group
    constexpr int kTailPerLane = kTailVec / 32;
    const int valid = max(0, min(128, T - row0));    // rows before T (< 128 here)
    const int g8 = valid >> 3;                        // whole 8-row groups by TMA
    const int tail0 = g8 << 3;                        // first row of the partial group
    auto swz = [&](int r, int c) {
        return dst + (c >> 3) * L::kChunkBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
    };
    uint4 vals[kTailPerLane];
#pragma unroll
    for (int u = 0; u < kTailPerLane; ++u) {
        const int idx = lane + 32 * u;
        const int r = tail0 + idx / kVecPerRow, c = idx % kVecPerRow;
        vals[u] = make_uint4(0u, 0u, 0u, 0u);
        if (r < valid)
            vals[u] = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(row0 + r) * row_stride +
                                                      static_cast<size_t>(col0) * E::kBytes + c * 16);
    }
#pragma unroll
    for (int u = 0; u < kTailPerLane; ++u) {
        const int idx = lane + 32 * u;
        const int r = tail0 + idx / kVecPerRow, c = idx % kVecPerRow;
        if (r < 128) *reinterpret_cast<uint4*>(swz(r, c)) = vals[u];
    }
    for (int idx = lane; idx < (128 - tail0 - 8) * kVecPerRow; idx += 32) {
        const int r = tail0 + 8 + idx / kVecPerRow, c = idx % kVecPerRow;
        *reinterpret_cast<uint4*>(swz(r, c)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        mbar_arrive_expect_tx(full, static_cast<uint32_t>(g8 * L::kChunks * 1024));
        for (int g = 0; g < g8; ++g) {
#pragma unroll
            for (int c = 0; c < L::kChunks; ++c)
                tma_load_2d(dst + c * L::kChunkBytes + g * 1024, map8, col0 + c * L::kChunkCols,
                            row0 + g * 8, full);
        }
    }
    __syncwarp();
}

// Whole warp: one 128-row tile into `dst`, completion signalled on `full`.
template <int D, class E>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, const CUtensorMap* map8,
                                          const uint8_t* src, int row0, int T, int row_stride,
                                          int col0, uint64_t* full, int lane) {
    using L = PrefillSmem<D, E>;
    if (row0 + 128 <= T) {
        if (lane == 0) {
            mbar_arrive_expect_tx(full, L::kTileBytes);
#pragma unroll
            for (int c = 0; c < L::kChunks; ++c)
                tma_load_2d(dst + c * L::kChunkBytes, map, col0 + c * L::kChunkCols, row0, full);
        }
        __syncwarp();
    } else {
        load_tile_ragged<D, E>(dst, map8, src, row0, T, row_stride, col0, full, lane);
    }
}

template <int D, class E>
__device__ __forceinline__ void store_row_zero(const PrefillParams& p, size_t out_row) {
    // zero is all-zero bits in both formats
    uint4* o4 = reinterpret_cast<uint4*>(p.out + out_row * (D * E::kBytes));
#pragma unroll
    for (int c = 0; c < D * E::kBytes / 16; ++c) o4[c] = make_uint4(0u, 0u, 0u, 0u);
    p.lse[out_row] = -INFINITY;
}

// kRes (bf16 only): the variant that serves the list's second part, the query
// blocks holding a row that sees few keys, with every role's per-item code
// also multiplying V by P's bf16 rounding residual (see kResidualMaxKeys); the
// main variant carries none of that code.  The host launches the residual
// variant right after the schedule build and the main variant as its
// programmatic dependent, so the short few-key items run beside the main
// part's longest ones instead of after its tail.
template <int D, class E, bool kRes>
__global__ void __launch_bounds__(kPrefillThreads, 1)
prefill_fwd_kernel(const __grid_constant__ PrefillMaps maps, const PrefillParams p) {
    static_assert(!(kRes && E::kFp8), "the residual variant is bf16 only");
    using L = PrefillSmem<D, E>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* q_full = bars + 0;  // [2]
    uint64_t* q_empty = bars + 2;
    uint64_t* k_full = bars + 3;
    uint64_t* k_empty = k_full + L::kStages;
    uint64_t* v_full = k_empty + L::kStages;
    uint64_t* v_empty = v_full + L::kStages;
    uint64_t* s_full = v_empty + L::kStages;  // [2]
    uint64_t* p_half = s_full + 2;         // [2], P of the tile's first 64 keys stored
    uint64_t* p_full = p_half + 2;         // [2], all of P stored
    uint64_t* o_done = p_full + 2;         // [2]
    uint64_t* item_full = o_done + 2;      // [2]
    uint64_t* item_empty = item_full + 2;  // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    volatile int* item_ring = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);  // [2]
    // the producer decodes each item once (cu_seqlens and the tile list are
    // global-memory reads) and publishes it here next to its index
    Item* item_slot = reinterpret_cast<Item*>(smem + L::kItems);                   // [2]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if constexpr (kRes) {
        // Wait for the schedule build, then let the main variant launch.  The
        // grid is one CTA per SM and the CTAs claim items from one counter, so
        // the first n_items CTAs serve every item between them; the others
        // leave before any set-up and hand their SM to the main variant at once.
        grid_dependency_wait();
        grid_launch_dependents();
        const int n_list = min(max(__ldcg(&p.hdr->n_tiles), 0), p.tile_capacity);
        const int n_main = min(max(__ldcg(&p.hdr->n_main), 0), n_list);
        if (static_cast<long long>(blockIdx.x) >= static_cast<long long>(n_list - n_main) * p.H) return;
    }

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(&q_full[x], 1);
            mbar_init(&s_full[x], 1);
            mbar_init(&p_half[x], 4);
            mbar_init(&p_full[x], 4);
            mbar_init(&o_done[x], 1);
            mbar_init(&item_full[x], 1);
            mbar_init(&item_empty[x], 1 + 8);  // the MMA lane and the eight softmax warps
        }
        mbar_init(q_empty, 1);
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tensormap(&maps.q);
        prefetch_tensormap(&maps.k);
        prefetch_tensormap(&maps.v);
    }
    if constexpr (!kRes) {
        // Straight after the schedule build (E4M3) the set-up above overlaps
        // the build and this wait covers everything below, which reads the
        // list it writes.  After the residual variant there is no wait here:
        // this grid launches only once every CTA of that variant is past its
        // own wait for the completed build, so the list is final and is read
        // through L2 (the header below, the entries in decode_item); the wait
        // for the residual variant's completion comes at the exit instead,
        // which keeps the stream's order for whatever follows.
        if (!p.after_residual) grid_dependency_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // this variant's part of the list as item indices (block index x H +
    // head): the main part [0, n_main H), the few-key part [n_main H, n_list H)
    const int n_list = min(max(__ldcg(&p.hdr->n_tiles), 0), p.tile_capacity);
    const int n_main = min(max(__ldcg(&p.hdr->n_main), 0), n_list);
    const int item0 = kRes ? n_main * p.H : 0;
    const int n_items = (kRes ? n_list - n_main : n_main) * p.H;
    int* counter = kRes ? &p.hdr->next_item_res : &p.hdr->next_item;
    const int group = p.H / p.H_kv;
    unsigned* status = &g_va_status;

    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer
        const int T_q = p.cu_q[p.batch], T_k = p.cu_k[p.batch];
        const int q_stride = p.H * D * E::kBytes, kv_stride = p.H_kv * D * E::kBytes;  // bytes
        uint32_t items_done = 0, q_issued[2] = {0, 0}, k_issued = 0, v_issued = 0, ring = 0;
        bool ok = true;
        for (;;) {
            // claim the next work item (longest first across the grid) and publish it
            int idx = -1;
            if (lane == 0) {
                const int t = atomicAdd(counter, 1);
                idx = t < n_items ? item0 + t : -1;
            }
            idx = __shfl_sync(0xffffffffu, idx, 0);
            Item it;
            if (idx >= 0) decode_item(p, idx, group, it);
            if (!(ok = mbar_wait_warp(&item_empty[ring & 1], ((ring >> 1) & 1) ^ 1, abort_flag, status)))
                break;
            if (lane == 0) {
                item_ring[ring & 1] = idx;
                if (idx >= 0) item_slot[ring & 1] = it;
                mbar_arrive(&item_full[ring & 1]);  // release: the slot's contents are visible
            }
            __syncwarp();
            ++ring;
            if (idx < 0) break;
            if (it.hi <= it.lo) continue;
            if (!(ok = mbar_wait_warp(q_empty, (items_done & 1) ^ 1, abort_flag, status))) break;
            ++items_done;
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                if (it.hi_h[x] > it.lo_h[x]) {
                    load_tile<D, E>(smem + L::kQ + x * L::kTileBytes, &maps.q, &maps.q8, p.q, it.q_row0 + x * kBlockM,
                                 T_q, q_stride, it.h * D, &q_full[x], lane);
                    ++q_issued[x];
                }
            }
            for (int kt = it.lo; kt < it.hi; ++kt) {
                const int s = k_issued % L::kStages;
                const uint32_t ph = (k_issued / L::kStages) & 1;
                if (!(ok = mbar_wait_warp(&k_empty[s], ph ^ 1, abort_flag, status))) break;
                load_tile<D, E>(smem + L::kK + s * L::kTileBytes, &maps.k, &maps.k8, p.k, it.k_row0 + kt * kBlockN,
                             T_k, kv_stride, it.hk * D, &k_full[s], lane);
                ++k_issued;
                if (!(ok = mbar_wait_warp(&v_empty[s], ph ^ 1, abort_flag, status))) break;
                load_tile<D, E>(smem + L::kV + s * L::kTileBytes, &maps.v, &maps.v8, p.v, it.k_row0 + kt * kBlockN,
                             T_k, kv_stride, it.hk * D, &v_full[s], lane);
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
            drain(&q_full[0], q_issued[0]);
            drain(&q_full[1], q_issued[1]);
            for (int s = 0; s < L::kStages; ++s) {
                const uint32_t nk = k_issued > (uint32_t)s ? (k_issued - s + L::kStages - 1) / L::kStages : 0;
                const uint32_t nv = v_issued > (uint32_t)s ? (v_issued - s + L::kStages - 1) / L::kStages : 0;
                drain(&k_full[s], nk);
                drain(&v_full[s], nv);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk =
                E::kFp8 ? idesc_e4m3_f32(128, kBlockN, false) : idesc_bf16_f32(128, kBlockN, false);
            constexpr uint32_t idesc_pv =
                E::kFp8 ? idesc_e4m3_f32(128, D, true) : idesc_bf16_f32(128, D, true);
            // one MMA step consumes 32 bytes of every operand row: 16 bf16 or 32 E4M3
            constexpr int kStepKeys = 32 / E::kBytes;
            // descriptors: one high word per operand kind, low words stepped by the
            // start-address field (16-byte units)
            static_assert(L::kBar < (1 << 18), "descriptor start-address field covers 256 KB");
            const uint64_t dq = smem_desc_sw128(smem_u32(smem + L::kQ), 16, 1024);
            const uint64_t dk = smem_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
            const uint64_t dv = smem_desc_sw128(smem_u32(smem + L::kV), L::kChunkBytes, 1024);
            const uint32_t q_lo = static_cast<uint32_t>(dq), q_hi = static_cast<uint32_t>(dq >> 32);
            const uint32_t k_lo = static_cast<uint32_t>(dk), k_hi = static_cast<uint32_t>(dk >> 32);
            const uint32_t v_lo = static_cast<uint32_t>(dv), v_hi = static_cast<uint32_t>(dv >> 32);
            uint32_t q_waits[2] = {0, 0}, p_waits[2] = {0, 0}, kv = 0, ring = 0;
            bool ok = true;

            auto issue_qk = [&](int x, int s) {
                const uint32_t qa = q_lo + ((x * L::kTileBytes) >> 4);
                const uint32_t kb = k_lo + ((s * L::kTileBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < L::kRowBytes / 32; ++kk) {
                    const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
                    if constexpr (E::kFp8)
                        mma_ss_lh_f8<idesc_qk>(tmem + L::tmem_s(x), qa + off, q_hi, kb + off, k_hi,
                                               kk > 0 ? 1u : 0u);
                    else
                        mma_ss_lh<idesc_qk>(tmem + L::tmem_s(x), qa + off, q_hi, kb + off, k_hi,
                                            kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[x]);
            };
            // O_x += P_x V.  Only the half's last PV of the item is committed to
            // o_done (the epilogue waits for it); earlier ones need no barrier of
            // their own: the S-ready commit of the next QK of the same half tracks
            // every MMA issued before it, this PV included.
            // Keys [64 part, 64 part + 64) of the tile (the part-th half of P); each
            // step reads 32 bytes of P per row (8 tensor-memory columns) and
            // kStepKeys rows of V.
            auto issue_pv = [&](int x, int s, bool first, bool last, int part) {
                const uint32_t vb = v_lo + ((s * L::kTileBytes) >> 4);
                constexpr int kSteps = (kBlockN / 2) / kStepKeys;
#pragma unroll
                for (int k4 = 0; k4 < kSteps; ++k4) {
                    const int kk = part * kSteps + k4;
                    const uint32_t vk = vb + ((kk * kStepKeys * 128) >> 4);
                    const uint32_t acc = (!first || kk > 0) ? 1u : 0u;
                    if constexpr (E::kFp8)
                        mma_ts_lh_f8<idesc_pv>(tmem + L::tmem_o(x), tmem + L::tmem_s(x) + kk * 8, vk,
                                               v_hi, acc);
                    else
                        mma_ts_lh<idesc_pv>(tmem + L::tmem_o(x), tmem + L::tmem_s(x) + kk * 8, vk,
                                            v_hi, acc);
                }
                if constexpr (kRes) {
                    // the same keys' residual P - bf16(P), stored 64 columns further on
#pragma unroll
                    for (int k4 = 0; k4 < kSteps; ++k4) {
                        const int kk = part * kSteps + k4;
                        const uint32_t vk = vb + ((kk * kStepKeys * 128) >> 4);
                        mma_ts_lh<idesc_pv>(tmem + L::tmem_o(x), tmem + L::tmem_s(x) + 64 + kk * 8,
                                            vk, v_hi, 1u);
                    }
                }
                if (last) mma_commit(&o_done[x]);
            };

            for (;;) {
                if (!(ok = mbar_wait(&item_full[ring & 1], (ring >> 1) & 1, abort_flag, status))) break;
                const int idx = item_ring[ring & 1];
                Item it;
                if (idx >= 0) it = item_slot[ring & 1];
                mbar_arrive(&item_empty[ring & 1]);
                ++ring;
                if (idx < 0) break;
                if (it.hi <= it.lo) continue;
                const int n = it.hi - it.lo;
                for (int x = 0; x < 2 && ok; ++x) {
                    if (it.hi_h[x] > it.lo_h[x])
                        ok = mbar_wait(&q_full[x], q_waits[x]++ & 1, abort_flag, status);
                }
                if (!ok) break;
                // prologue: S for the first key tile
                {
                    const int s = kv % L::kStages;
                    if (!(ok = mbar_wait(&k_full[s], (kv / L::kStages) & 1, abort_flag, status))) break;
                    tc_fence_after();
                    for (int x = 0; x < 2; ++x)
                        if (takes_part(it, x, it.lo)) issue_qk(x, s);
                    mma_commit(&k_empty[s]);
                    if (n == 1) mma_commit(q_empty);  // last reader of Q issued
                }
                bool first_pv[2] = {true, true};
                for (int j = 0; j < n && ok; ++j) {
                    const int kt = it.lo + j;
                    const uint32_t kv_j = kv + j, kv_n = kv + j + 1;
                    const int s = kv_j % L::kStages, s_n = kv_n % L::kStages;
                    const bool has_next = j + 1 < n;
                    bool next_k_ready = false;
                    if (!(ok = mbar_wait(&v_full[s], (kv_j / L::kStages) & 1, abort_flag, status))) break;
                    for (int x = 0; x < 2 && ok; ++x) {
                        if (takes_part(it, x, kt)) {
                            const uint32_t pw = p_waits[x]++ & 1;
                            if (!(ok = mbar_wait(&p_half[x], pw, abort_flag, status))) break;
                            tc_fence_after();
                            issue_pv(x, s, first_pv[x], false, 0);
                            if (!(ok = mbar_wait(&p_full[x], pw, abort_flag, status))) break;
                            tc_fence_after();
                            issue_pv(x, s, first_pv[x], kt + 1 == it.hi_h[x], 1);
                            first_pv[x] = false;
                        }
                        if (has_next && takes_part(it, x, kt + 1)) {
                            if (!next_k_ready) {
                                if (!(ok = mbar_wait(&k_full[s_n], (kv_n / L::kStages) & 1, abort_flag, status)))
                                    break;
                                tc_fence_after();
                                next_k_ready = true;
                            }
                            issue_qk(x, s_n);
                        }
                    }
                    if (!ok) break;
                    if (has_next) {
                        if (!next_k_ready) {
                            // every tile of the union has a taker; this wait only keeps
                            // the ring's phases in step if that ever changes
                            if (!(ok = mbar_wait(&k_full[s_n], (kv_n / L::kStages) & 1, abort_flag, status)))
                                break;
                        }
                        mma_commit(&k_empty[s_n]);
                        // the QKs of the last key tile are issued: Q may be reloaded as
                        // soon as they complete, while the last softmax and PV run
                        if (j + 2 == n) mma_commit(q_empty);
                    }
                    mma_commit(&v_empty[s]);
                }
                if (!ok) break;
                kv += n;
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int x = warp >> 2;                    // which half of the query block
        const int quarter = warp & 3;               // TMEM lane quarter this warp may access
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t sbase = tmem + lane_addr + L::tmem_s(x);
        const uint32_t obase = tmem + lane_addr + L::tmem_o(x);
        uint32_t s_waits = 0, o_waits = 0, ring = 0;
        bool ok = true;
        for (;;) {
            if (!(ok = mbar_wait_warp(&item_full[ring & 1], (ring >> 1) & 1, abort_flag, status))) break;
            const int idx = item_ring[ring & 1];
            Item it;
            if (idx >= 0) it = item_slot[ring & 1];
            __syncwarp();
            if (lane == 0) mbar_arrive(&item_empty[ring & 1]);
            ++ring;
            if (idx < 0) break;
            const int i = it.qb * kBlockQ + x * kBlockM + row_in_tile;
            const bool row_valid = i < it.L_q;
            int lo, hi;
            row_key_interval(i, it.L_q, it.L_k, p.causal != 0, p.window, lo, hi);
            const size_t out_row = static_cast<size_t>(it.q_row0 + x * kBlockM + row_in_tile) * p.H + it.h;
            if (it.hi_h[x] <= it.lo_h[x]) {
                if (row_valid) store_row_zero<D, E>(p, out_row);
                continue;
            }
            // keys every row of this warp sees: tiles inside [warp_lo, warp_hi] need no mask
            const int warp_lo = __reduce_max_sync(0xffffffffu, lo);
            const int warp_hi = __reduce_min_sync(0xffffffffu, hi);
            // l: row sum of P (for the logsumexp); l_norm: the normaliser of O, the
            // row sum of P as the PV product sees it (see the tile-maximum term below)
            float m_ref = -INFINITY, l = 0.f, l_norm = 0.f;
            for (int kt = it.lo_h[x]; kt < it.hi_h[x]; ++kt) {
                const bool first_tile = kt == it.lo_h[x];
                if (!(ok = mbar_wait_warp(&s_full[x], s_waits++ & 1, abort_flag, status))) break;
                tc_fence_after();
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
                    for (int c = 0; c < 32; ++c) {
                        s[c] = __uint_as_float(r0[c]);
                        s[32 + c] = __uint_as_float(r1[c]);
                        s[64 + c] = __uint_as_float(r2[c]);
                        s[96 + c] = __uint_as_float(r3[c]);
                    }
                }
                const int key0 = kt * kBlockN;
                if (!(warp_lo <= key0 && key0 + kBlockN - 1 <= warp_hi)) {
                    // column c is visible iff lo <= key0 + c <= hi: one unsigned range
                    // check per element against this row's bounds relative to the tile
                    // (a row that sees no key gets an offset no column reaches)
                    const bool any = hi >= lo;
                    const int c_lo = any ? lo - key0 : (1 << 30);
                    const unsigned span = any ? static_cast<unsigned>(hi - lo) : 0u;
#pragma unroll
                    for (int c = 0; c < kBlockN; ++c)
                        s[c] = (static_cast<unsigned>(c - c_lo) <= span) ? s[c] : -INFINITY;
                }
                // row max as a tree of three-input maxima (eight short chains)
                static_assert(kBlockN == 128, "the max tree covers 128 columns");
                float mv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mv[e] = max3f(s[e], s[8 + e], s[16 + e]);
#pragma unroll
                for (int c = 24; c < 120; c += 16)
#pragma unroll
                    for (int e = 0; e < 8; ++e) mv[e] = max3f(mv[e], s[c + e], s[c + 8 + e]);
#pragma unroll
                for (int e = 0; e < 8; ++e) mv[e] = fmaxf(mv[e], s[120 + e]);
                const float mx = max3f(max3f(mv[0], mv[1], mv[2]), max3f(mv[3], mv[4], mv[5]),
                                       fmaxf(mv[6], mv[7]));
                const float m_tile = mx * p.scale_log2;  // -inf stays -inf
                const float m_cand = fmaxf(m_ref, m_tile);
                const bool want = first_tile || (m_cand > m_ref + kRescaleThreshold);
                const bool move = __any_sync(0xffffffffu, want);
                float alpha = 1.f;
                if (move) {
                    alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - m_cand);
                    m_ref = m_cand;
                }
                const float m_sub = (m_ref == -INFINITY) ? 0.f : m_ref;
                // The PV product multiplies P as rounded to the input format, the row
                // sum takes P itself; where one weight dominates a row, the dominant
                // weight's rounding would then scale O by up to 2^-9.  So the
                // normaliser also takes the rounding of each tile's largest P (the
                // same FMA and exp2 the loop below applies to that score; 0 for a
                // row that sees no key of the tile).  The residual variant multiplies
                // P's rounding residual too, so there the normaliser is P's sum.
                float tmax_round = 0.f;
                if constexpr (!E::kFp8 && !kRes) {
                    const float pt = ex2_approx(__fmaf_rn(mx, p.scale_log2, -m_sub));
                    tmax_round = __bfloat162float(__float2bfloat16_rn(pt)) - pt;
                }
                // P = 2^(s * scale_log2 - m_ref) into S_x in the input format (bf16
                // pairs or E4M3 quadruples), 64 keys at a time; the first 64 are handed over on their own so
                // their PV starts while the second half is computed.  S_x's previous P
                // was consumed by the PV issued before this QK.
                // (pairs of columns through the packed f32x2 FMA and add)
                const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
                const uint64_t neg2 = f2_pack(-m_sub, -m_sub);
                uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};  // eight partial sums, as pairs
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if constexpr (E::kFp8) {
                        // four E4M3 values per column: keys 64 half + [0, 64) in 16 columns
                        uint32_t pk[16];
#pragma unroll
                        for (int c = 0; c < 64; c += 4) {
                            float x0, x1, x2, x3;
                            f2_unpack(f2_fma(f2_pack(s[half * 64 + c], s[half * 64 + c + 1]), scale2, neg2),
                                      x0, x1);
                            f2_unpack(f2_fma(f2_pack(s[half * 64 + c + 2], s[half * 64 + c + 3]), scale2,
                                             neg2),
                                      x2, x3);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
                            sum2[(c >> 2) & 3] = f2_add(sum2[(c >> 2) & 3], f2_add(f2_pack(p0, p1), f2_pack(p2, p3)));
                            pk[c / 4] = pack_e4m3x4(p0, p1, p2, p3);
                        }
                        tmem_st16(sbase + half * 16, pk);
                    } else if constexpr (kRes) {
                        // P as bf16 plus its residual P - bf16(P) (exact in f32) as bf16,
                        // 64 columns further on, over scores already read; 16 keys at a
                        // time
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8) {
                            const int k0 = half * 64 + q8 * 16;
                            uint32_t pk[8], rk[8];
#pragma unroll
                            for (int c = 0; c < 16; c += 2) {
                                float x0, x1;
                                f2_unpack(f2_fma(f2_pack(s[k0 + c], s[k0 + c + 1]), scale2, neg2), x0, x1);
                                const uint64_t pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
                                sum2[(c >> 1) & 3] = f2_add(sum2[(c >> 1) & 3], pp);
                                float p0, p1;
                                f2_unpack(pp, p0, p1);
                                const uint32_t b2 = pack_bf16x2(p0, p1);
                                pk[c / 2] = b2;
                                float r0, r1;
                                f2_unpack(f2_sub(pp, bf16x2_to_f2(b2)), r0, r1);
                                rk[c / 2] = pack_bf16x2(r0, r1);
                            }
                            tmem_st8(sbase + half * 32 + q8 * 8, pk);
                            tmem_st8(sbase + 64 + half * 32 + q8 * 8, rk);
                        }
                    } else {
                        uint32_t pk[32];
#pragma unroll
                        for (int c = 0; c < 64; c += 2) {
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(s[half * 64 + c], s[half * 64 + c + 1]), scale2, neg2),
                                      x0, x1);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            sum2[(c >> 1) & 3] = f2_add(sum2[(c >> 1) & 3], f2_pack(p0, p1));
                            pk[c / 2] = pack_bf16x2(p0, p1);
                        }
                        tmem_st32(sbase + half * 32, pk);
                    }
                    if (half == 0) {
                        if (!first_tile && move) {
                            // O_x holds every earlier P V: they were issued before this
                            // tile's QK, whose completion the S-ready barrier observed.
                            // Rescale it before any P of this tile reaches the MMA warp.
#pragma unroll
                            for (int c = 0; c < D / 32; ++c) {
                                uint32_t r[32];
                                tmem_ld32(obase + c * 32, r);
                                tmem_wait_ld();
#pragma unroll
                                for (int e = 0; e < 32; ++e)
                                    r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                                tmem_st32(obase + c * 32, r);
                            }
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&p_half[x]);
                    }
                }
                float sums[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) f2_unpack(sum2[e], sums[2 * e], sums[2 * e + 1]);
                const float tile_sum = ((sums[0] + sums[1]) + (sums[2] + sums[3])) +
                                       ((sums[4] + sums[5]) + (sums[6] + sums[7]));
                l = l * alpha + tile_sum;
                l_norm = l_norm * alpha + (tile_sum + tmax_round);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[x]);
            }
            if (!ok) break;
            // epilogue: wait for the half's last P V (the only one committed to
            // o_done), then O / l and logsumexp
            if (!(ok = mbar_wait_warp(&o_done[x], o_waits++ & 1, abort_flag, status))) break;
            tc_fence_after();
            // O / l, times v_scale / o_scale for E4M3 (V's dequantization and the
            // output's quantization folded into one factor)
            const float inv_l = l_norm > 0.f ? p.out_mul / l_norm : 0.f;
            {
                // every column block in flight before a single wait
                uint32_t r[D / 32][32];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) tmem_ld32(obase + c * 32, r[c]);
                tmem_wait_ld();
                // Through a per-warp shared-memory slice, one 64-byte column block (32
                // bf16 or 64 E4M3 values) at a time, so that each global store
                // instruction writes eight rows x 64 contiguous bytes instead of 16
                // bytes of 32 different rows.  The 16-byte chunk e of slice row r sits
                // at position e ^ ((r >> 1) & 3): both the row-per-lane writes and the
                // 8-row reads are conflict-free.
                uint8_t* stage = smem + L::kStage + warp * 2048;
                const int row_base = x * kBlockM + quarter * 32;  // first tile row of this warp
                constexpr int kBlocks = L::kRowBytes / 64;
                auto o_at = [&](int col) { return __uint_as_float(r[col >> 5][col & 31]) * inv_l; };
#pragma unroll
                for (int c = 0; c < kBlocks; ++c) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint4 w;
                        if constexpr (E::kFp8) {
                            const int c0 = c * 64 + e * 16;
                            w.x = pack_e4m3x4(o_at(c0 + 0), o_at(c0 + 1), o_at(c0 + 2), o_at(c0 + 3));
                            w.y = pack_e4m3x4(o_at(c0 + 4), o_at(c0 + 5), o_at(c0 + 6), o_at(c0 + 7));
                            w.z = pack_e4m3x4(o_at(c0 + 8), o_at(c0 + 9), o_at(c0 + 10), o_at(c0 + 11));
                            w.w = pack_e4m3x4(o_at(c0 + 12), o_at(c0 + 13), o_at(c0 + 14), o_at(c0 + 15));
                        } else {
                            const int c0 = c * 32 + e * 8;
                            w.x = pack_bf16x2(o_at(c0 + 0), o_at(c0 + 1));
                            w.y = pack_bf16x2(o_at(c0 + 2), o_at(c0 + 3));
                            w.z = pack_bf16x2(o_at(c0 + 4), o_at(c0 + 5));
                            w.w = pack_bf16x2(o_at(c0 + 6), o_at(c0 + 7));
                        }
                        *reinterpret_cast<uint4*>(stage + lane * 64 + ((e ^ ((lane >> 1) & 3)) << 4)) = w;
                    }
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = i * 8 + (lane >> 2), ch = lane & 3;
                        const uint4 v = *reinterpret_cast<const uint4*>(stage + rr * 64 + ((ch ^ ((rr >> 1) & 3)) << 4));
                        if (it.qb * kBlockQ + row_base + rr < it.L_q) {
                            const size_t orow = static_cast<size_t>(it.q_row0 + row_base + rr) * p.H + it.h;
                            *reinterpret_cast<uint4*>(p.out + orow * L::kRowBytes + c * 64 + ch * 16) = v;
                        }
                    }
                    __syncwarp();
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
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if constexpr (!kRes) grid_dependency_wait();
}

}  // namespace va
