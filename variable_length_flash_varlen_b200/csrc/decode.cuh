// Decode-shape forward (one query row per sequence): split-K streaming of
// K/V from HBM on CUDA cores, then a combine pass that merges the per-split
// partial results through their logsumexp.
//
// One CTA owns (sequence b, up to kDecodeHeads query heads of one KV head,
// one split of at most `chunk` keys), so every K/V row it reads serves all of
// those heads at once (boostr 0.2.0 varlen_attention.rs, VarLenAttentionOps
// docs, "GQA key/value head mapping": kv_head = q_head / (H / H_kv)).  Each K
// or V row is read by D/8 lanes with one 16-byte non-caching load each.
//
// Split s keeps (m_s, l_s, O_s): the max of its base-2 scaled scores, the sum
// of 2^(score - m_s) and the unnormalised sum of 2^(score - m_s) v.  The
// combine takes M = max m_s, L = sum 2^(m_s - M) l_s,
// O = sum 2^(m_s - M) O_s / L and logsumexp = (M + log2 L) ln 2 — the same
// rescaling the online softmax of realizar 0.8.4 attention.rs (IMP-111
// online_softmax) applies tile by tile, applied once across splits.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"
#include "status.cuh"

namespace va {

constexpr int kDecodeThreads = 128;
constexpr int kDecodeHeads = 4;         // query heads per CTA
constexpr int kDecodeMaxChunk = 1024;   // keys per split (shared-memory score buffer)
constexpr int kDecodeUnroll = 8;        // K/V rows in flight per row group

struct DecodeParams {
    const int* cu_q;
    const int* cu_k;
    int batch, H, H_kv, causal, window;
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    float* part_o;   // [batch, H, n_split_max, D]
    float* part_ml;  // [batch, H, n_split_max, 2]
    int n_split_max;
    int chunk;
    float scale_log2;
    __nv_bfloat16* out;
    float* lse;
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* ptr) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(ptr));
    return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Visible key interval of the single query row of sequence b.
__device__ __forceinline__ void decode_row_interval(const DecodeParams& p, int b, int& L_q,
                                                   int& lo, int& hi) {
    L_q = p.cu_q[b + 1] - p.cu_q[b];
    const int L_k = p.cu_k[b + 1] - p.cu_k[b];
    row_key_interval(0, L_q, L_k, p.causal != 0, p.window, lo, hi);
}

template <int D>
__global__ void __launch_bounds__(kDecodeThreads)
decode_split_kernel(const DecodeParams p) {
    constexpr int LPR = D / 8;            // lanes per K/V row
    constexpr int RPW = 32 / LPR;         // rows per warp
    constexpr int NGRP = (kDecodeThreads / 32) * RPW;  // row groups per CTA
    __shared__ float sc[kDecodeHeads][kDecodeMaxChunk];
    __shared__ float red[NGRP][kDecodeHeads][D];
    __shared__ float s_ml[kDecodeHeads][2];

    const int b = blockIdx.x, split = blockIdx.z;
    const int G = p.H / p.H_kv;
    const int groups_per_kv = (G + kDecodeHeads - 1) / kDecodeHeads;
    const int hk = blockIdx.y / groups_per_kv;
    const int g0 = (blockIdx.y % groups_per_kv) * kDecodeHeads;
    const int nh = min(kDecodeHeads, G - g0);
    const int h0 = hk * G + g0;  // first query head of this CTA

    int L_q, lo, hi;
    decode_row_interval(p, b, L_q, lo, hi);
    if (L_q <= 0 || hi < lo) return;
    const int k_begin = lo + split * p.chunk;
    if (k_begin > hi) return;
    const int k_end = min(hi + 1, k_begin + p.chunk);
    const int n = k_end - k_begin;
    const size_t krow0 = static_cast<size_t>(p.cu_k[b]);
    const int q_tok = p.cu_q[b];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp * RPW + lane / LPR;
    const int sub = lane % LPR;

    // query slices, pre-scaled into base-2 score units
    float qv[kDecodeHeads][8];
#pragma unroll
    for (int g = 0; g < kDecodeHeads; ++g) {
        if (g < nh) {
            const uint4 u = *reinterpret_cast<const uint4*>(
                p.q + (static_cast<size_t>(q_tok) * p.H + h0 + g) * D + sub * 8);
            bf16x8_to_f32(u, qv[g]);
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[g][e] *= p.scale_log2;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[g][e] = 0.f;
        }
    }

    // ---- scores: one row group per key, D/8 lanes per row.  The trip count
    // is the same for every lane (warp shuffles below need the whole warp).
    for (int base0 = 0; base0 < n; base0 += NGRP * kDecodeUnroll) {
        const int base = base0 + grp;
        uint4 kr[kDecodeUnroll];
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const int kk = base + u * NGRP;
            if (kk < n)
                kr[u] = ld_stream_v4(p.k + ((krow0 + k_begin + kk) * p.H_kv + hk) * D + sub * 8);
            else
                kr[u] = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            float kf[8];
            bf16x8_to_f32(kr[u], kf);
            float dot[kDecodeHeads];
#pragma unroll
            for (int g = 0; g < kDecodeHeads; ++g) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) a = fmaf(qv[g][e], kf[e], a);
                dot[g] = a;
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) {
#pragma unroll
                for (int g = 0; g < kDecodeHeads; ++g) dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], o);
            }
            const int kk = base + u * NGRP;
            if (sub == 0 && kk < n) {
#pragma unroll
                for (int g = 0; g < kDecodeHeads; ++g) sc[g][kk] = dot[g];
            }
        }
    }
    __syncthreads();

    // ---- per head: max, exponentials, sum (warp g owns head g)
    if (warp < nh) {
        float m = -INFINITY;
        for (int x = lane; x < n; x += 32) m = fmaxf(m, sc[warp][x]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int x = lane; x < n; x += 32) {
            const float e = ex2_approx(sc[warp][x] - m);
            sc[warp][x] = e;
            l += e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) {
            s_ml[warp][0] = m;
            s_ml[warp][1] = l;
        }
    }
    __syncthreads();

    // ---- P V
    float acc[kDecodeHeads][8];
#pragma unroll
    for (int g = 0; g < kDecodeHeads; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
    for (int base0 = 0; base0 < n; base0 += NGRP * kDecodeUnroll) {
        const int base = base0 + grp;
        uint4 vr[kDecodeUnroll];
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const int kk = base + u * NGRP;
            if (kk < n)
                vr[u] = ld_stream_v4(p.v + ((krow0 + k_begin + kk) * p.H_kv + hk) * D + sub * 8);
            else
                vr[u] = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const int kk = base + u * NGRP;
            if (kk < n) {
                float vf[8];
                bf16x8_to_f32(vr[u], vf);
#pragma unroll
                for (int g = 0; g < kDecodeHeads; ++g) {
                    const float w = sc[g][kk];
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(w, vf[e], acc[g][e]);
                }
            }
        }
    }
#pragma unroll
    for (int g = 0; g < kDecodeHeads; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) red[grp][g][sub * 8 + e] = acc[g][e];
    __syncthreads();
    for (int x = threadIdx.x; x < nh * D; x += kDecodeThreads) {
        const int g = x / D, d = x % D;
        float t = 0.f;
#pragma unroll
        for (int r = 0; r < NGRP; ++r) t += red[r][g][d];
        const size_t slot = (static_cast<size_t>(b) * p.H + h0 + g) * p.n_split_max + split;
        p.part_o[slot * D + d] = t;
        if (d == 0) {
            p.part_ml[slot * 2 + 0] = s_ml[g][0];
            p.part_ml[slot * 2 + 1] = s_ml[g][1];
        }
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
    for (int s = 0; s < ns; ++s) M = fmaxf(M, p.part_ml[(slot0 + s) * 2]);
    float Lsum = 0.f, o = 0.f;
    for (int s = 0; s < ns; ++s) {
        const float w = ex2_approx(p.part_ml[(slot0 + s) * 2] - M);
        Lsum = fmaf(w, p.part_ml[(slot0 + s) * 2 + 1], Lsum);
        o = fmaf(w, p.part_o[(slot0 + s) * D + d], o);
    }
    p.out[out_row * D + d] = __float2bfloat16_rn(o / Lsum);
    if (d == 0) p.lse[out_row] = (M + log2f(Lsum)) * 0.69314718055994530942f;
}

}  // namespace va
