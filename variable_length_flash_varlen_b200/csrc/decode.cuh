// Decode-shape forward (one query row per sequence): K/V streamed from HBM by
// TMA into a shared-memory ring and consumed by warp-level tensor-core tiles
// with a single-pass online softmax, then a combine pass that merges
// per-split partial results through their logsumexp.
//
// Work unit: (sequence b, group of up to kDecodeHeads query heads sharing one
// KV head, split of `chunk` keys).  Every K/V row streamed serves all heads of
// the group at once (boostr 0.2.0 varlen_attention.rs, VarLenAttentionOps
// docs, "GQA key/value head mapping": kv_head = q_head / (H / H_kv)).  The
// heads of the group are the 16 rows of an m16n8k16 product: S = Q K^T over
// 16 keys, then O += P V, so one key costs two tensor-core instructions per
// warp instead of ~45 scalar ones (rows past the group's head count are zero
// and discarded).  Persistent CTAs (one per SM) claim units from a counter.
// Per CTA: warp 4 streams 64-key tiles of K and V (TMA, 128-byte swizzle;
// 8-row boxes and plain loads for a tile that runs past the end of the packed tensor) into a
// ring; warps 0-3 each take 16 keys of every tile and keep, per head, a
// running max m (base-2 scaled scores, moved lazily by more than 2^8), a
// running sum l and an unnormalised output.  At the end of a unit the four
// warps are merged and the split's (m, l, O) written out.
//
// The combine takes M = max m_s, L = sum 2^(m_s - M) l_s,
// O = sum 2^(m_s - M) O_s / N with N the same sum over the splits'
// normalisers (row sums of P as rounded for the product), and logsumexp =
// (M + log2 L) ln 2 — the same
// rescaling the online softmax of realizar 0.8.4 attention.rs (IMP-111
// online_softmax) applies tile by tile, applied once across splits.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"
#include "status.cuh"

namespace va {

constexpr int kDecodeHeads = 16;         // query heads per unit (mma rows)
constexpr int kDecodeWarpKeys = 16;      // keys per compute warp per tile
constexpr int kDecodeComputeWarps = 4;
constexpr int kDecodeTileKeys = kDecodeWarpKeys * kDecodeComputeWarps;  // keys per ring stage
constexpr int kDecodeThreads = 32 * (kDecodeComputeWarps + 1);
constexpr int kDecodeMaxDefaultChunk = 4096;  // default split: the largest power of two
constexpr int kDecodeMinDefaultChunk = 256;   // in this range giving kDecodeUnitsPerSm
constexpr int kDecodeUnitsPerSm = 8;          // units per SM (unless the caller chooses)
constexpr float kDecodeRescaleThreshold = 8.0f;

struct DecodeParams {
    const int* cu_q;
    const int* cu_k;
    const int* seqused_k;  // optional key counts of a capacity-strided cache (else NULL)
    int batch, H, H_kv, causal, window;
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    float* part_o;   // [batch, H, n_split_max, D]
    float* part_ml;  // [batch, H, n_split_max, 4]: m, row sum of P, normaliser (rounded P's sum), -
    int* counter;    // unit counter, zero before the launch
    int n_split_max;
    int chunk;
    int n_units;     // batch * kv-head groups * n_split_max
    float scale_log2;
    __nv_bfloat16* out;
    float* lse;
};

// Shared memory of the streaming kernel.  A K or V tile is D/64 column
// halves of [64 keys][64 columns] bf16 (128-byte rows, 128-byte swizzle: the
// 16-byte chunk c of row r sits at chunk position c ^ (r & 7)); every tile
// starts on a 1024-byte boundary so that pattern holds for absolute addresses.
template <int D>
struct DecodeSmem {
    static constexpr int kStages = D == 64 ? 10 : 5;
    static constexpr int kHalfBytes = kDecodeTileKeys * 128;
    static constexpr int kTileBytes = kDecodeTileKeys * D * 2;
    static constexpr int kK = 0;
    static constexpr int kV = kK + kStages * kTileBytes;
    static constexpr int kRed = kV + kStages * kTileBytes;           // [warps][heads][D + 3] f32
    static constexpr int kRedBytes = kDecodeComputeWarps * kDecodeHeads * (D + 3) * 4;
    static constexpr int kBar = kRed + kRedBytes;                    // full[S], empty[S], item_full[2], item_empty[2]
    static constexpr int kMisc = kBar + (2 * kStages + 4) * 8;
    static constexpr int kBytes = kMisc + 16;                        // abort flag, item ring[2]
    static constexpr int kAlloc = kBytes + 1024;
};

// Visible key interval of the single query row of sequence b.
__device__ __forceinline__ void decode_row_interval(const DecodeParams& p, int b, int& L_q,
                                                   int& lo, int& hi) {
    L_q = p.cu_q[b + 1] - p.cu_q[b];
    const int L_k = seq_key_count(p.cu_k, p.seqused_k, b);
    row_key_interval(0, L_q, L_k, p.causal != 0, p.window, lo, hi);
}

struct DecodeUnit {
    int b, hk, g0, nh, split, k_begin, n_keys;
    bool residual;  // the row sees few keys: P's bf16 rounding residual is multiplied in too
};

// A query that sees at most this many keys puts most of its softmax weight on
// a few of them, and the bf16 rounding of P (2^-9 relative per weight) no
// longer averages out; its units also multiply V by the residual
// P - bf16(P), rounded to bf16 (two more tensor-core products per 16 keys).
constexpr int kDecodeResidualMaxKeys = 256;

// Unit u -> its sequence, head group and key range; false if it holds no key.
__device__ __forceinline__ bool decode_unit(const DecodeParams& p, int u, DecodeUnit& w) {
    const int G = p.H / p.H_kv;
    const int gpk = (G + kDecodeHeads - 1) / kDecodeHeads;
    w.split = u % p.n_split_max;
    const int rest = u / p.n_split_max;
    const int grp = rest % (p.H_kv * gpk);
    w.b = rest / (p.H_kv * gpk);
    w.hk = grp / gpk;
    w.g0 = (grp % gpk) * kDecodeHeads;
    w.nh = min(kDecodeHeads, G - w.g0);
    int L_q, lo, hi;
    decode_row_interval(p, w.b, L_q, lo, hi);
    if (L_q <= 0 || hi < lo) return false;
    w.k_begin = lo + w.split * p.chunk;
    if (w.k_begin > hi) return false;
    w.residual = hi - lo + 1 <= kDecodeResidualMaxKeys;
    w.n_keys = min(hi + 1, w.k_begin + p.chunk) - w.k_begin;
    return true;
}

template <int D>
__global__ void __launch_bounds__(kDecodeThreads, 1)
decode_stream_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmK8, const __grid_constant__ CUtensorMap tmV8,
                     const DecodeParams p) {
    using L = DecodeSmem<D>;
    constexpr int S = L::kStages;
    constexpr int KC = D / 16;       // 16-column steps of the score product
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* empty = full + S;
    uint64_t* item_full = empty + S;
    uint64_t* item_empty = item_full + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc);
    volatile int* item_ring = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);  // [2]
    float* red = reinterpret_cast<float*>(smem + L::kRed);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned* status = &g_va_status;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDecodeComputeWarps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&item_full[s], 1);
            mbar_init(&item_empty[s], kDecodeComputeWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kDecodeComputeWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        const int T_k = p.cu_k[p.batch];
        const int stride = p.H_kv * D;
        uint32_t issued = 0, ring = 0;
        bool ok = true;
        for (;;) {
            int u = -1;
            DecodeUnit w;
            // claim units until one holds keys (or none are left)
            for (;;) {
                int t = 0;
                if (lane == 0) t = atomicAdd(p.counter, 1);
                t = __shfl_sync(0xffffffffu, t, 0);
                if (t >= p.n_units) break;
                if (decode_unit(p, t, w)) {
                    u = t;
                    break;
                }
            }
            if (!(ok = mbar_wait_warp(&item_empty[ring & 1], ((ring >> 1) & 1) ^ 1, abort_flag, status)))
                break;
            if (lane == 0) {
                item_ring[ring & 1] = u;
                mbar_arrive(&item_full[ring & 1]);
            }
            __syncwarp();
            ++ring;
            if (u < 0) break;
            const int k0 = p.cu_k[w.b] + w.k_begin;
            const int n_tiles = (w.n_keys + kDecodeTileKeys - 1) / kDecodeTileKeys;
            for (int t = 0; t < n_tiles; ++t, ++issued) {
                const int s = issued % S;
                if (!(ok = mbar_wait_warp(&empty[s], ((issued / S) & 1) ^ 1, abort_flag, status)))
                    break;
                uint8_t* kt = smem + L::kK + s * L::kTileBytes;
                uint8_t* vt = smem + L::kV + s * L::kTileBytes;
                // both tiles complete one phase of full[s]: expect their bytes together
                const int row0 = k0 + t * kDecodeTileKeys;
                if (row0 + kDecodeTileKeys <= T_k) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[s], 2 * L::kTileBytes);
#pragma unroll
                        for (int h = 0; h < D / 64; ++h) {
                            tma_load_2d(kt + h * L::kHalfBytes, &tmK, w.hk * D + h * 64, row0, &full[s]);
                            tma_load_2d(vt + h * L::kHalfBytes, &tmV, w.hk * D + h * 64, row0, &full[s]);
                        }
                    }
                    __syncwarp();
                } else {
                    // The same swizzled layout, rows at or past T_k zero: whole 8-row
                    // groups before T_k by TMA in 8-row boxes (a box written at a
                    // 1024-byte-aligned offset has the swizzle phase of those rows of a
                    // full box), the one partial group by plain loads all in flight at
                    // once, the rest zero-filled.  (The maps' row extent is only an
                    // upper bound of T_k, so no box may reach past it.)
                    constexpr int kVecPerRow = D / 8;
                    constexpr int kTailPerLane = 8 * kVecPerRow / 32;
                    const int valid = max(0, min(kDecodeTileKeys, T_k - row0));
                    const int g8 = valid >> 3, tail0 = g8 << 3;
                    auto swz = [](int r, int c) {
                        return (c >> 3) * L::kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
                    };
                    uint4 kvals[kTailPerLane], vvals[kTailPerLane];
#pragma unroll
                    for (int u = 0; u < kTailPerLane; ++u) {
                        const int idx = lane + 32 * u;
                        const int r = tail0 + idx / kVecPerRow, c = idx % kVecPerRow;
                        kvals[u] = make_uint4(0u, 0u, 0u, 0u);
                        vvals[u] = kvals[u];
                        if (r < valid) {
                            const size_t off = static_cast<size_t>(row0 + r) * stride + w.hk * D + c * 8;
                            kvals[u] = *reinterpret_cast<const uint4*>(p.k + off);
                            vvals[u] = *reinterpret_cast<const uint4*>(p.v + off);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < kTailPerLane; ++u) {
                        const int idx = lane + 32 * u;
                        const int r = tail0 + idx / kVecPerRow, c = idx % kVecPerRow;
                        if (r < kDecodeTileKeys) {
                            *reinterpret_cast<uint4*>(kt + swz(r, c)) = kvals[u];
                            *reinterpret_cast<uint4*>(vt + swz(r, c)) = vvals[u];
                        }
                    }
                    for (int idx = lane; idx < (kDecodeTileKeys - tail0 - 8) * kVecPerRow; idx += 32) {
                        const int r = tail0 + 8 + idx / kVecPerRow, c = idx % kVecPerRow;
                        *reinterpret_cast<uint4*>(kt + swz(r, c)) = make_uint4(0u, 0u, 0u, 0u);
                        *reinterpret_cast<uint4*>(vt + swz(r, c)) = make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(2 * g8 * (D / 64) * 1024));
                        for (int g = 0; g < g8; ++g) {
#pragma unroll
                            for (int h = 0; h < D / 64; ++h) {
                                tma_load_2d(kt + h * L::kHalfBytes + g * 1024, &tmK8, w.hk * D + h * 64,
                                            row0 + g * 8, &full[s]);
                                tma_load_2d(vt + h * L::kHalfBytes + g * 1024, &tmV8, w.hk * D + h * 64,
                                            row0 + g * 8, &full[s]);
                            }
                        }
                    }
                    __syncwarp();
                }
            }
            if (!ok) break;
        }
        if (!ok && lane == 0 && issued > 0) {
            // abandoned: wait (bounded) for the copies in flight before exiting
            const unsigned long long t0 = global_timer_ns();
            for (int s = 0; s < S; ++s) {
                const uint32_t n = issued > (uint32_t)s ? (issued - s + S - 1) / S : 0;
                if (n == 0) continue;
                while (!mbar_try_wait(&full[s], (n - 1) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------- compute
    const int g = lane >> 2, tq = lane & 3;
    // ldmatrix row addresses (byte offsets inside a tile) of this lane.  K
    // (scores, plain): matrices (keys 0-7 | 8-15) x (columns 0-7 | 8-15) of
    // a 16-column step, lane -> key (lane & 7) + 8 (lane >> 4), chunk
    // (lane >> 3) & 1.  V (P V, transposed): lane -> key (lane & 7) +
    // 8 ((lane >> 3) & 1), chunk lane >> 4.
    const int key_k = warp * kDecodeWarpKeys + (lane & 7) + ((lane >> 4) << 3);
    const int key_v = warp * kDecodeWarpKeys + (lane & 7) + (((lane >> 3) & 1) << 3);
    const int xk = ((lane >> 3) & 1) ^ (lane & 7);
    const int xv = (lane >> 4) ^ (lane & 7);
    uint32_t offk[4], offv[4];   // by (16-column step) mod 4: chunk pair 2j, 2j + 1
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        offk[j] = key_k * 128 + (((2 * j) ^ xk) << 4);
        offv[j] = key_v * 128 + (((2 * j) ^ xv) << 4);
    }
    const uint32_t k_smem = smem_u32(smem + L::kK), v_smem = smem_u32(smem + L::kV);

    uint32_t consumed = 0, ring = 0;
    for (;;) {
        if (!mbar_wait_warp(&item_full[ring & 1], (ring >> 1) & 1, abort_flag, status)) break;
        const int u = item_ring[ring & 1];
        __syncwarp();
        if (lane == 0) mbar_arrive(&item_empty[ring & 1]);
        ++ring;
        if (u < 0) break;
        DecodeUnit w;
        decode_unit(p, u, w);
        const int h0 = w.hk * (p.H / p.H_kv) + w.g0;
        const int q_tok = p.cu_q[w.b];

        // Q of the group as mma row operands (rows past nh zero), unscaled bf16
        uint32_t qa[KC][4];
        {
            const uint32_t* q_lo = reinterpret_cast<const uint32_t*>(
                p.q + (static_cast<size_t>(q_tok) * p.H + h0 + g) * D);
            const uint32_t* q_hi = reinterpret_cast<const uint32_t*>(
                p.q + (static_cast<size_t>(q_tok) * p.H + h0 + g + 8) * D);
            const bool lo_ok = g < w.nh, hi_ok = g + 8 < w.nh;
#pragma unroll
            for (int kc = 0; kc < KC; ++kc) {
                qa[kc][0] = lo_ok ? q_lo[kc * 8 + tq] : 0u;
                qa[kc][1] = hi_ok ? q_hi[kc * 8 + tq] : 0u;
                qa[kc][2] = lo_ok ? q_lo[kc * 8 + 4 + tq] : 0u;
                qa[kc][3] = hi_ok ? q_hi[kc * 8 + 4 + tq] : 0u;
            }
        }
        float o[D / 8][4];
#pragma unroll
        for (int nb = 0; nb < D / 8; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;
        // rows g, g + 8: reference max, row sum of P, normaliser (sum of the P the
        // product multiplies)
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, ln[2] = {0.f, 0.f};

        const int n_tiles = (w.n_keys + kDecodeTileKeys - 1) / kDecodeTileKeys;
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t, ++consumed) {
            const int s = consumed % S;
            if (!(ok = mbar_wait_warp(&full[s], (consumed / S) & 1, abort_flag, status))) break;
            const uint32_t kt = k_smem + s * L::kTileBytes, vt = v_smem + s * L::kTileBytes;

            // scores of this warp's 16 keys: sc[n][.] covers keys 8n + 2tq (+1)
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kc = 0; kc < KC; ++kc) {
                uint32_t b[4];
                ldsm_x4(kt + (kc >> 2) * L::kHalfBytes + offk[kc & 3], b);
                mma_16816(sc[0], qa[kc], b[0], b[1]);
                mma_16816(sc[1], qa[kc], b[2], b[3]);
            }
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[n][e] *= p.scale_log2;
            const int key0 = t * kDecodeTileKeys + warp * kDecodeWarpKeys;
            if (key0 + kDecodeWarpKeys > w.n_keys) {
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (key0 + 8 * n + 2 * tq + (e & 1) >= w.n_keys) sc[n][e] = -INFINITY;
            }
            float mt[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mt[r] = fmaxf(fmaxf(sc[0][2 * r], sc[0][2 * r + 1]), fmaxf(sc[1][2 * r], sc[1][2 * r + 1]));
                mt[r] = fmaxf(mt[r], __shfl_xor_sync(0xffffffffu, mt[r], 1));
                mt[r] = fmaxf(mt[r], __shfl_xor_sync(0xffffffffu, mt[r], 2));
            }
            const bool up0 = mt[0] > m[0] + kDecodeRescaleThreshold;
            const bool up1 = mt[1] > m[1] + kDecodeRescaleThreshold;
            if (__any_sync(0xffffffffu, up0 || up1)) {
                float alpha[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const bool up = r == 0 ? up0 : up1;
                    alpha[r] = 1.f;
                    if (up) {
                        alpha[r] = (m[r] == -INFINITY) ? 0.f : ex2_approx(m[r] - mt[r]);
                        m[r] = mt[r];
                    }
                    l[r] *= alpha[r];
                    ln[r] *= alpha[r];
                }
#pragma unroll
                for (int nb = 0; nb < D / 8; ++nb) {
                    o[nb][0] *= alpha[0];
                    o[nb][1] *= alpha[0];
                    o[nb][2] *= alpha[1];
                    o[nb][3] *= alpha[1];
                }
            }
            const float mu0 = (m[0] == -INFINITY) ? 0.f : m[0];
            const float mu1 = (m[1] == -INFINITY) ? 0.f : m[1];
            float pr[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                pr[n][0] = ex2_approx(sc[n][0] - mu0);
                pr[n][1] = ex2_approx(sc[n][1] - mu0);
                pr[n][2] = ex2_approx(sc[n][2] - mu1);
                pr[n][3] = ex2_approx(sc[n][3] - mu1);
            }
            const uint32_t pa[4] = {pack_bf16x2(pr[0][0], pr[0][1]), pack_bf16x2(pr[0][2], pr[0][3]),
                                    pack_bf16x2(pr[1][0], pr[1][1]), pack_bf16x2(pr[1][2], pr[1][3])};
            // bf16 bits are the upper half of the f32 bits
            auto lo_of = [](uint32_t b2) { return __uint_as_float(b2 << 16); };
            auto hi_of = [](uint32_t b2) { return __uint_as_float(b2 & 0xFFFF0000u); };
            l[0] += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
            l[1] += (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
            if (!w.residual) {
                // the normaliser takes P as rounded to bf16, the values the PV product
                // multiplies, so a dominant weight's rounding cancels in O / l; the
                // logsumexp keeps the sum of P itself
                ln[0] = add_bf16x2_f32(pa[2], add_bf16x2_f32(pa[0], ln[0]));
                ln[1] = add_bf16x2_f32(pa[3], add_bf16x2_f32(pa[1], ln[1]));
#pragma unroll
                for (int db = 0; db < D / 16; ++db) {
                    uint32_t b[4];
                    ldsm_x4_trans(vt + (db >> 2) * L::kHalfBytes + offv[db & 3], b);
                    mma_16816(o[2 * db], pa, b[0], b[1]);
                    mma_16816(o[2 * db + 1], pa, b[2], b[3]);
                }
            } else {
                ln[0] += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
                ln[1] += (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
                // f32 minus its bf16 rounding is exact
                const uint32_t ra[4] = {
                    pack_bf16x2(pr[0][0] - lo_of(pa[0]), pr[0][1] - hi_of(pa[0])),
                    pack_bf16x2(pr[0][2] - lo_of(pa[1]), pr[0][3] - hi_of(pa[1])),
                    pack_bf16x2(pr[1][0] - lo_of(pa[2]), pr[1][1] - hi_of(pa[2])),
                    pack_bf16x2(pr[1][2] - lo_of(pa[3]), pr[1][3] - hi_of(pa[3]))};
#pragma unroll
                for (int db = 0; db < D / 16; ++db) {
                    uint32_t b[4];
                    ldsm_x4_trans(vt + (db >> 2) * L::kHalfBytes + offv[db & 3], b);
                    mma_16816(o[2 * db], pa, b[0], b[1]);
                    mma_16816(o[2 * db + 1], pa, b[2], b[3]);
                    mma_16816(o[2 * db], ra, b[0], b[1]);
                    mma_16816(o[2 * db + 1], ra, b[2], b[3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (!ok) break;

        // merge the four warps through shared memory
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
            ln[r] += __shfl_xor_sync(0xffffffffu, ln[r], 1);
            ln[r] += __shfl_xor_sync(0xffffffffu, ln[r], 2);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int row = g + 8 * r;
            if (row < w.nh) {
                float* dst = red + (warp * kDecodeHeads + row) * (D + 3);
#pragma unroll
                for (int nb = 0; nb < D / 8; ++nb) {
                    dst[nb * 8 + 2 * tq] = o[nb][2 * r];
                    dst[nb * 8 + 2 * tq + 1] = o[nb][2 * r + 1];
                }
                if (tq == 0) {
                    dst[D] = m[r];
                    dst[D + 1] = l[r];
                    dst[D + 2] = ln[r];
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecodeComputeWarps) : "memory");
        for (int idx = threadIdx.x; idx < w.nh * D; idx += 32 * kDecodeComputeWarps) {
            const int hh = idx / D, d = idx % D;
            float M = -INFINITY;
#pragma unroll
            for (int ww = 0; ww < kDecodeComputeWarps; ++ww)
                M = fmaxf(M, red[(ww * kDecodeHeads + hh) * (D + 3) + D]);
            float acc = 0.f, lsum = 0.f, nsum = 0.f;
#pragma unroll
            for (int ww = 0; ww < kDecodeComputeWarps; ++ww) {
                const float* src = red + (ww * kDecodeHeads + hh) * (D + 3);
                const float f = (src[D] == -INFINITY) ? 0.f : ex2_approx(src[D] - M);
                acc = fmaf(src[d], f, acc);
                lsum = fmaf(src[D + 1], f, lsum);
                nsum = fmaf(src[D + 2], f, nsum);
            }
            const size_t slot = (static_cast<size_t>(w.b) * p.H + h0 + hh) * p.n_split_max + w.split;
            p.part_o[slot * D + d] = acc;
            if (d == 0) {
                p.part_ml[slot * 4 + 0] = M;
                p.part_ml[slot * 4 + 1] = lsum;
                p.part_ml[slot * 4 + 2] = nsum;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecodeComputeWarps) : "memory");
    }
}

template <int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const DecodeParams p) {
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
    int L_q, lo, hi;
    decode_row_interval(p, b, L_q, lo, hi);
    if (L_q <= 0) return;
    const size_t out_row = static_cast<size_t>(p.cu_q[b]) * p.H + h;
    const int d = threadIdx.x;
    if (hi < lo) {
        p.out[out_row * D + d] = __float2bfloat16_rn(0.f);
        if (d == 0) p.lse[out_row] = -INFINITY;
        return;
    }
    const int ns = (hi - lo + 1 + p.chunk - 1) / p.chunk;
    const size_t slot0 = (static_cast<size_t>(b) * p.H + h) * p.n_split_max;
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, p.part_ml[(slot0 + s) * 4]);
    float Lsum = 0.f, Nsum = 0.f, o = 0.f;
    for (int s = 0; s < ns; ++s) {
        const float w = ex2_approx(p.part_ml[(slot0 + s) * 4] - M);
        Lsum = fmaf(w, p.part_ml[(slot0 + s) * 4 + 1], Lsum);
        Nsum = fmaf(w, p.part_ml[(slot0 + s) * 4 + 2], Nsum);
        o = fmaf(w, p.part_o[(slot0 + s) * D + d], o);
    }
    p.out[out_row * D + d] = __float2bfloat16_rn(o / Nsum);
    if (d == 0) p.lse[out_row] = (M + log2f(Lsum)) * 0.69314718055994530942f;
}

}  // namespace va
