// dequant_math.cuh -- the exact FP8 -> fp32 quotient RN(q / s) used by the
// dequantize and fake-quantize kernels.
//
// The method is Markstein's residual-correction division (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990; also his "IA-64 and Elementary
// Functions", 2000): a quotient estimate from the rounded reciprocal, its
// exact residual from one fused multiply-add, and one correction step.
// Every FP8 value is (1 + j/8) * 2^a.  With r = RN(1/s),
//     y0 = RN(q * r);  e = RN(q - s * y0) (fma);  y = RN(y0 + e * r) (fma)
// The general theorem asks for conditions that are not checked here;
// instead, for the FP8 dividends this library has, the result is verified
// to equal the IEEE quotient for every code as long as no step leaves the
// normal range: tests/c/recip_division_exhaustive.c checks the 8 FP8
// significands against all 2^23 scale significands.  That holds for |s| in
// [2^-100, 2^101); other scales use the per-element IEEE division.
#pragma once

#include <cstdint>

#include "fp8q_device.cuh"

namespace fp8q {

// |s| in [2^-100, 2^101): r, q * r, the residual and the result all stay normal.
__device__ __forceinline__ bool scale_fast_ok(float s) {
    const uint32_t ex = (__float_as_uint(s) >> 23) & 0xFFu;
    return ex >= 27u && ex <= 227u;
}

// True when any of the 4 codes in w is an E5M2 Inf/NaN code (exponent field all ones).
__device__ __forceinline__ bool e5m2_has_special(uint32_t w) {
    return (((w & 0x7C7C7C7Cu) + 0x04040404u) & 0x80808080u) != 0u;
}

// Two codes (low 16 bits of c2) -> two exact quotients RN(q / s), from
// r2 = {RN(1/s)} x2 and ns2 = {-s} x2:
//   y0 = q * r;  e = q - s * y0 (fma);  y = y0 + e * r (fma)
// For q = +-0 the last fma would give +0 for -0, so the sign is taken from
// y0, which carries the quotient's sign for every q.
template <int FMT>
__device__ __forceinline__ float2 dequant2_fast(uint32_t c2, uint64_t r2, uint64_t ns2) {
    const float2 a = fp8x2_to_float2<FMT>(c2);
    const uint64_t q2 = f32x2(a.x, a.y);
    const uint64_t y0 = mul_f32x2(q2, r2);
    const uint64_t e = fma_f32x2(y0, ns2, q2);
    const float2 y = f32x2_split(fma_f32x2(e, r2, y0));
    const float2 z = f32x2_split(y0);
    return make_float2(copysignf(y.x, z.x), copysignf(y.y, z.y));
}

template <int FMT>
__device__ __forceinline__ float2 dequant2_div(uint32_t c2, float s) {
    const float2 a = fp8x2_to_float2<FMT>(c2);
    return make_float2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s));
}

}  // namespace fp8q
