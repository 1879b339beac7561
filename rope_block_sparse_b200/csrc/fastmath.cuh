// Packed fp32 pair arithmetic (f32x2 instructions of sm_100a) used by the
// attention softmax, a three-input max, and an FMA-pipe exp2 (self-test only).
#pragma once

#include <cstdint>

namespace h3a {

// Packed pairs of fp32 (one 64-bit register, two lanes of the FMA pipe).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// max(a, b, c) in one instruction (three-input max.f32 of sm_100a).
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x for a pair on the FMA pipe instead of the MUFU unit: x = n + f with
// n = round(x) (adding 1.5 * 2^23 leaves n in the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f from a degree-3 polynomial minimising the relative
// error on [-1/2, 1/2] (Remez exchange, max relative error 7.5e-5, far below
// the 2^-9 of the bf16 P it feeds; coefficients from csrc/fit_exp2_poly.py);
// 2^n is added into the exponent field.  Inputs are clamped to >= -126 (below
// that the result is at most 2^-126, i.e. zero for P).
__device__ __forceinline__ uint64_t exp2_poly_pair(uint64_t x) {
    float x0, x1;
    f2_split(x, x0, x1);
    x = f2(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
    const uint64_t shifter = f2(12582912.0f, 12582912.0f);
    const uint64_t t = f2_add(x, shifter);
    const uint64_t f = f2_sub(x, f2_sub(t, shifter));
    uint64_t p = f2_fma(f2(0.0551716685f, 0.0551716685f), f, f2(0.242611125f, 0.242611125f));
    p = f2_fma(p, f, f2(0.693260968f, 0.693260968f));
    p = f2_fma(p, f, f2(0.999928057f, 0.999928057f));
    float p0, p1, t0, t1;
    f2_split(p, p0, p1);
    f2_split(t, t0, t1);
    // the low bits of t hold n; shifted into the exponent field (mod 2^32)
    return f2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
              __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

}  // namespace h3a
