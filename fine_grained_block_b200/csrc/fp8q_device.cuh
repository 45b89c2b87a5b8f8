// fp8q_device.cuh -- device-side building blocks of libfp8q (sm_100a).
//
// Arithmetic fixed by the pages (PyTorch-FP8 page s1.2-s1.3, s4.1-s4.2;
// mixed-precision handbook "FP8 training"):
//   s = fp32(MAX / max(amax, 1e-12f))      IEEE division, round to nearest
//   q = fp8(fp32(x * s)), saturating, round to nearest even
//   y = fp32(decode(q) / s)                 IEEE division, round to nearest
// Every rounding step is spelled out with an explicit-rounding intrinsic or a
// PTX instruction with a stated rounding mode, so the result does not depend
// on compiler contraction or fast-math flags.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp8q {

constexpr int kE4M3 = 0;
constexpr int kE5M2 = 1;

// Largest finite value of each format (PyTorch-FP8 page, s1.2 table).
template <int FMT>
__host__ __device__ constexpr float fmt_max() { return FMT == kE4M3 ? 448.0f : 57344.0f; }

// amax clamp (handbook per_block clamp(min=1e-12) on an fp32 tensor).
constexpr float kAmaxEps = 1e-12f;

// ---------------------------------------------------------------------------
// scale
// ---------------------------------------------------------------------------

// s = MAX / max(amax, eps) with one IEEE round-to-nearest division.
template <int FMT>
__device__ __forceinline__ float scale_from_amax(float amax) {
    return __fdiv_rn(fmt_max<FMT>(), fmaxf(amax, kAmaxEps));
}

// ---------------------------------------------------------------------------
// casts
// ---------------------------------------------------------------------------

// Two fp32 values -> two FP8 codes in the low 16 bits; `lo` lands in the low
// byte (the lower address in memory).  cvt.rn.satfinite: round to nearest
// even, out-of-range values (and +-Inf) saturate to +-MAX, NaN stays NaN.
template <int FMT>
__device__ __forceinline__ uint32_t cvt_fp8x2(float lo, float hi) {
    uint16_t r;
    if constexpr (FMT == kE4M3) {
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    } else {
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    }
    return r;
}

// Two FP8 codes (low 16 bits of `c2`, low byte first) -> two exact fp32.
// FP8 -> f16 is exact for both formats (every E4M3/E5M2 value is an f16
// value), and f16 -> f32 is exact.
template <int FMT>
__device__ __forceinline__ float2 fp8x2_to_float2(uint32_t c2) {
    uint32_t h;
    const uint16_t c = static_cast<uint16_t>(c2);
    if constexpr (FMT == kE4M3) {
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
    } else {
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h) : "h"(c));
    }
    float lo, hi;
    asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"(static_cast<uint16_t>(h & 0xFFFFu)));
    asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"(static_cast<uint16_t>(h >> 16)));
    return make_float2(lo, hi);
}

// Two fp32 -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// bf16 halves of a 32-bit word -> fp32 (exact: bf16 is the top half of fp32).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------------------
// amax
// ---------------------------------------------------------------------------

// Running max of |x| over packed bf16 pairs.  The sign bits are cleared and
// max.bf16x2 keeps the larger value of each half (a NaN operand yields the
// other operand, so NaN never wins).  Exact: no rounding is involved.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t acc, uint32_t w) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w & 0x7FFF7FFFu));
    return r;
}

// Larger of the two halves of a packed |bf16| pair, as fp32.
__device__ __forceinline__ float bf16x2_hmax(uint32_t m) {
    return fmaxf(bf16_lo(m), bf16_hi(m));
}

template <int WIDTH>
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int off = WIDTH / 2; off > 0; off >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
    return v;
}

// ---------------------------------------------------------------------------
// memory access
// ---------------------------------------------------------------------------

// Streaming 16-byte load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Streaming stores (written once, evict-first in L2).
__device__ __forceinline__ void st_stream(uint2* p, uint2 v) {
    asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ void st_stream(uint4* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void st_stream(uint32_t* p, uint32_t v) {
    asm volatile("st.global.cs.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// fp32 -> orderable unsigned (valid for values >= +0, which is all amax ever is).
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
    atomicMax(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

}  // namespace fp8q
