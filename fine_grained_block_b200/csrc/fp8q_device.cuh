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

// MX block scale (handbook, FP8 training notes: Blackwell's MX formats give
// every 32 elements one shared power-of-two scale).  Returns s = 2^k and sets
// `byte` to its E8M0 encoding 127 - k (the exponent of the dequant multiplier
// 2^-k; E8M0 byte 0xFF is NaN).
//   rule 0 (fit): the largest k with max(amax, eps) * 2^k <= MAX;
//   rule 1 (OCP MX): k = emax - floor(log2(max(amax, eps))).
// MAX is 1.75 * 2^emax in both formats (emax 8 and 15), so for
// a = m * 2^e with m in [1, 2), rule 1 is k = emax - e and rule 0 takes one
// less when m > 1.75 -- integer work on the bits of a.  The eps clamp keeps a
// normal, so k lies in [-120, 55] and 2^k is a normal fp32.  An infinite amax
// has no fitting power of two: s = 1 and the NaN byte.
template <int FMT>
__device__ __forceinline__ float mx_scale(float amax, int rule, uint8_t& byte) {
    constexpr int kEmax = FMT == kE4M3 ? 8 : 15;
    const uint32_t b = __float_as_uint(fmaxf(amax, kAmaxEps));
    const int e = static_cast<int>(b >> 23) - 127;
    if (e == 128) {
        byte = 0xFFu;
        return 1.0f;
    }
    const int k = kEmax - e - ((rule == 0 && (b & 0x7FFFFFu) > 0x600000u) ? 1 : 0);
    byte = static_cast<uint8_t>(127 - k);
    return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

// The dequant multiplier of an E8M0 byte: 2^(byte - 127) as an fp32 (byte 0
// is the subnormal 2^-127), NaN for byte 0xFF.
__device__ __forceinline__ float e8m0_to_float(uint32_t byte) {
    if (byte == 0xFFu) return __uint_as_float(0x7FC00000u);
    return byte == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(byte << 23);
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

// Running max of |x| over packed bf16 pairs with one instruction per pair:
// max.xorsign.abs takes the larger magnitude (its sign bit is the xor of the
// inputs' signs and is cleared at the end by bf16x2_absmax_finish).  A NaN
// operand yields the other operand.  Exact.
__device__ __forceinline__ uint32_t xabsmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ float bf16x2_absmax_finish(uint32_t m) {
    return bf16x2_hmax(m & 0x7FFF7FFFu);
}

// ---------------------------------------------------------------------------
// packed fp32 pairs (sm_100 f32x2 arithmetic: two IEEE round-to-nearest
// results per instruction, denormals kept)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ float2 f32x2_split(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return make_float2(lo, hi);
}

__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// A packed bf16 pair (lo element in the low half) scaled by s2 = {s, s} in
// fp32 and cast to two FP8 codes (low 16 bits, lo code in the low byte):
// q = fp8(fp32(x * s)) for both elements.
template <int FMT>
__device__ __forceinline__ uint32_t scale_cast_bf16x2(uint32_t w, uint64_t s2) {
    const float2 p = f32x2_split(mul_f32x2(f32x2(bf16_lo(w), bf16_hi(w)), s2));
    return cvt_fp8x2<FMT>(p.x, p.y);
}

template <int FMT>
__device__ __forceinline__ uint32_t scale_cast_f32x2(uint32_t a, uint32_t b, uint64_t s2) {
    const float2 p = f32x2_split(mul_f32x2(f32x2(__uint_as_float(a), __uint_as_float(b)), s2));
    return cvt_fp8x2<FMT>(p.x, p.y);
}

// ---------------------------------------------------------------------------
// memory access
// ---------------------------------------------------------------------------

// 32-byte vector (one 256-bit access per lane).
struct V32 {
    uint32_t w[8];
};

__device__ __forceinline__ V32 ld32_stream(const void* p) {
    V32 v;
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
                   "=r"(v.w[6]), "=r"(v.w[7])
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st32_stream(void* p, const V32& v) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]),
                    "r"(v.w[6]), "r"(v.w[7])
                 : "memory");
}

__device__ __forceinline__ V32 v32_zero() {
    V32 v;
#pragma unroll
    for (int k = 0; k < 8; ++k) v.w[k] = 0u;
    return v;
}

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
