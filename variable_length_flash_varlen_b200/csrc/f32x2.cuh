// Packed f32 pair arithmetic (sm_100a): two lanes' worth of FMA-pipe work per
// instruction, used by the element-wise softmax and gradient phases.
#pragma once

#include <cstdint>

namespace va {

// Packed pairs of f32 in one 64-bit register (lo, hi): one instruction of the
// f32x2 forms does two lanes' worth of FMA-pipe work, which halves the issue
// slots of the element-wise softmax arithmetic.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// A packed bf16 pair (low half = first value) widened to an f32 pair:
// the bf16 bits are the upper half of the f32 bits.
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t b2) {
    return f2_pack(__uint_as_float(b2 << 16), __uint_as_float(b2 & 0xFFFF0000u));
}
// max of three (one instruction)
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

}  // namespace va
