// dequant.cu -- FP8 dequantization kernels.
//
// PyTorch-FP8 page, s4.1 (divide by the scale to restore the value) and s4.2
// quantize() (.to(dtype) / scale): y = fp32(decode(q) / s), the correctly
// rounded IEEE quotient, then (bf16 output) one more round-to-nearest-even to
// bf16.
//
// The quotient is formed without a division per element.  Each thread takes
// r = RN(1/s) once for its group of codes and then, per element,
//     y0 = RN(q * r);  e = RN(q - s * y0) (fma);  y = RN(y0 + e * r) (fma).
// Every FP8 value is (1 + j/8) * 2^a, so with no step leaving the normal range
// the scheme is exact for all codes iff it is exact for the 8 mantissas of q
// against every one of the 2^23 mantissas of s -- 8 * 2^23 cases, all checked
// exhaustively by tests/c/recip_division_exhaustive.c.  The normal-range
// condition holds for |s| in [2^-100, 2^101), which covers every scale the
// quantizers produce except for amax above ~2^108; other scales, and E5M2
// Inf codes (whose fma residual would be Inf - Inf), take the per-element IEEE
// division instead.
//
// Each thread turns one group of codes into one 16- or 32-byte output vector
// (8 or 16 codes for bf16 output, 4 or 8 for fp32).  Consecutive lanes
// therefore read consecutive code groups and write consecutive vectors, so
// both the loads and the stores of a warp are contiguous.
//
// MX codes (1x32 blocks, E8M0 scale bytes) need no division: the value is
// decode(q) * 2^(byte - 127), one exact multiplication except at the ends of
// the fp32 range.

#include <algorithm>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "launch_util.h"
#include "dequant_math.cuh"
#include "lane_vec.cuh"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
// Code groups loaded per trip per thread.
#ifndef FP8Q_DEQ_UNROLL
#define FP8Q_DEQ_UNROLL 4
#endif
constexpr int kUnroll = FP8Q_DEQ_UNROLL;

template <int NW>
__device__ __forceinline__ void unpack_codes(const typename CodeWords<NW>::T& c, uint32_t* w);
template <>
__device__ __forceinline__ void unpack_codes<1>(const uint32_t& c, uint32_t* w) { w[0] = c; }
template <>
__device__ __forceinline__ void unpack_codes<2>(const uint2& c, uint32_t* w) { w[0] = c.x; w[1] = c.y; }
template <>
__device__ __forceinline__ void unpack_codes<4>(const uint4& c, uint32_t* w) {
    w[0] = c.x; w[1] = c.y; w[2] = c.z; w[3] = c.w;
}

__device__ __forceinline__ void store_words(void* p, const Words<4>& v) {
    st_stream(static_cast<uint4*>(p), make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]));
}
__device__ __forceinline__ void store_words(void* p, const Words<8>& v) {
    V32 o;
#pragma unroll
    for (int k = 0; k < 8; ++k) o.w[k] = v.w[k];
    st32_stream(p, o);
}

// One lane's group of codes -> one OB-byte output vector (OUT 0 = fp32, 1 = bf16).
template <int OUT, int OB>
struct DOut {
    static constexpr int kOutElem = OUT == 0 ? 4 : 2;
    static constexpr int kCodes = OB / kOutElem;
    static constexpr int kCodeWords = kCodes / 4;
    using In = typename CodeWords<kCodeWords>::T;
    using Out = Words<OB / 4>;

    template <int FMT>
    static __device__ __forceinline__ void put(Out& o, int pair, float2 y) {
        if (OUT == 1) {
            o.w[pair] = pack_bf16x2(y.x, y.y);
        } else {
            o.w[2 * pair] = __float_as_uint(y.x);
            o.w[2 * pair + 1] = __float_as_uint(y.y);
        }
    }

    template <int FMT>
    static __device__ __forceinline__ Out convert(const In& cin, float s) {
        uint32_t cw[kCodeWords];
        unpack_codes<kCodeWords>(cin, cw);
        bool fast = scale_fast_ok(s);
        if (FMT == kE5M2) {
#pragma unroll
            for (int k = 0; k < kCodeWords; ++k) fast = fast && !e5m2_has_special(cw[k]);
        }
        Out o;
        if (fast) {
            const float r = __frcp_rn(s);
            const uint64_t r2 = f32x2(r, r);
            const uint64_t ns2 = f32x2(-s, -s);
#pragma unroll
            for (int k = 0; k < kCodeWords; ++k) {
                put<FMT>(o, 2 * k, dequant2_fast<FMT>(cw[k] & 0xFFFFu, r2, ns2));
                put<FMT>(o, 2 * k + 1, dequant2_fast<FMT>(cw[k] >> 16, r2, ns2));
            }
        } else {
#pragma unroll
            for (int k = 0; k < kCodeWords; ++k) {
                put<FMT>(o, 2 * k, dequant2_div<FMT>(cw[k] & 0xFFFFu, s));
                put<FMT>(o, 2 * k + 1, dequant2_div<FMT>(cw[k] >> 16, s));
            }
        }
        return o;
    }

    // MX: y = RN(decode(q) * m), m = 2^(byte - 127).  The product of an FP8
    // value and a power of two is exact unless it leaves the fp32 normal
    // range, where the one rounding of mul.rn (no flush to zero) is the
    // rounding of the real product.
    template <int FMT>
    static __device__ __forceinline__ Out multiply(const In& cin, float m) {
        uint32_t cw[kCodeWords];
        unpack_codes<kCodeWords>(cin, cw);
        const uint64_t m2 = f32x2(m, m);
        Out o;
#pragma unroll
        for (int k = 0; k < kCodeWords; ++k) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 a = fp8x2_to_float2<FMT>(h ? (cw[k] >> 16) : (cw[k] & 0xFFFFu));
                put<FMT>(o, 2 * k + h, f32x2_split(mul_f32x2(f32x2(a.x, a.y), m2)));
            }
        }
        return o;
    }
};

__device__ __forceinline__ uint32_t ld_codes(const uint32_t* p) {
    return __ldcs(reinterpret_cast<const unsigned int*>(p));
}
__device__ __forceinline__ uint2 ld_codes(const uint2* p) { return __ldcs(p); }
__device__ __forceinline__ uint4 ld_codes(const uint4* p) { return __ldcs(p); }

// One code -> fp32 (for tails and the general kernel).
template <int FMT>
__device__ __forceinline__ float decode1(uint8_t c) { return fp8x2_to_float2<FMT>(c).x; }

// Per-tensor (MODE 0) and 1x128 (MODE 1, cols % 128 == 0) over a flat range
// of ngroups code groups.  Each CTA owns kThreads x kUnroll consecutive groups
// and issues all its loads before converting; a per-tensor tail of < kCodes
// codes goes to CTA 0.
template <int FMT, int OUT, int OB, int MODE>
__global__ void __launch_bounds__(kThreads)
k_dequant_flat(const typename DOut<OUT, OB>::In* __restrict__ q, int64_t ngroups,
               const uint8_t* __restrict__ q_tail, int tail_n, const float* __restrict__ scales,
               typename DOut<OUT, OB>::Out* __restrict__ y, void* __restrict__ y_tail) {
    pdl_enter();
    using D = DOut<OUT, OB>;
    constexpr int kGroupsPerBlock = 128 / D::kCodes;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads * kUnroll + threadIdx.x;
    const float s0 = (MODE == 0) ? scales[0] : 0.0f;
    typename D::In c[kUnroll];
    float s[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t g = base + u * kThreads;
        const bool ok = g < ngroups;
        c[u] = ok ? ld_codes(q + g) : typename D::In{};
        s[u] = (MODE == 0) ? s0 : (ok ? scales[g / kGroupsPerBlock] : 1.0f);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t g = base + u * kThreads;
        if (g < ngroups) store_words(y + g, D::template convert<FMT>(c[u], s[u]));
    }
    if (MODE == 0 && blockIdx.x == 0 && threadIdx.x < tail_n) {
        const float v = __fdiv_rn(decode1<FMT>(q_tail[threadIdx.x]), s0);
        if (OUT == 0) static_cast<float*>(y_tail)[threadIdx.x] = v;
        else static_cast<uint16_t*>(y_tail)[threadIdx.x] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
    }
}

// 128x128 (cols % 128 == 0): one CTA per tile, one scale per CTA.  A tile row
// is 128 codes = kGroupsPerRow groups; the CTA sweeps the tile's 128 rows.
template <int FMT, int OUT, int OB>
__global__ void __launch_bounds__(kThreads)
k_dequant_128x128(const typename DOut<OUT, OB>::In* __restrict__ q, const float* __restrict__ scales,
                  typename DOut<OUT, OB>::Out* __restrict__ y, int64_t rows, int64_t cols) {
    pdl_enter();
    using D = DOut<OUT, OB>;
    constexpr int kGroupsPerRow = 128 / D::kCodes;
    constexpr int kRowsPerPass = kThreads / kGroupsPerRow;
    constexpr int kPasses = 128 / kRowsPerPass;
    constexpr int kTileUnroll = 4;  // passes per batch of loads
    static_assert(kPasses % kTileUnroll == 0, "the unrolled passes must stay inside the tile");
    const int64_t tiles_c = cols >> 7;
    const int64_t tr = blockIdx.x / tiles_c;
    const int64_t tc = blockIdx.x - tr * tiles_c;
    const float s = scales[blockIdx.x];
    const int64_t groups_per_tensor_row = cols / D::kCodes;
    const int64_t r0 = tr * 128 + threadIdx.x / kGroupsPerRow;
    const int64_t g0 = r0 * groups_per_tensor_row + tc * kGroupsPerRow + threadIdx.x % kGroupsPerRow;
#pragma unroll
    for (int p0 = 0; p0 < kPasses; p0 += kTileUnroll) {
        typename D::In c[kTileUnroll];
#pragma unroll
        for (int u = 0; u < kTileUnroll; ++u) {
            const int64_t r = r0 + (p0 + u) * kRowsPerPass;
            c[u] = (r < rows) ? ld_codes(q + g0 + (p0 + u) * kRowsPerPass * groups_per_tensor_row)
                              : typename D::In{};
        }
#pragma unroll
        for (int u = 0; u < kTileUnroll; ++u) {
            const int64_t r = r0 + (p0 + u) * kRowsPerPass;
            if (r < rows)
                store_words(y + g0 + (p0 + u) * kRowsPerPass * groups_per_tensor_row,
                            D::template convert<FMT>(c[u], s));
        }
    }
}

// Any layout, element by element (ragged widths).  mode 1: 1x128, 2: 128x128.
template <int FMT, int OUT>
__global__ void __launch_bounds__(kThreads)
k_dequant_general(const uint8_t* __restrict__ q, int64_t rows, int64_t cols, int mode,
                  const float* __restrict__ scales, void* __restrict__ y) {
    pdl_enter();
    const int64_t n = rows * cols;
    const int64_t nbc = (cols + 127) / 128;
    const int br = (mode == 2) ? 128 : 1;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * kThreads) {
        const int64_t r = i / cols, c = i - (i / cols) * cols;
        const float s = (mode == 0) ? scales[0] : scales[(r / br) * nbc + c / 128];
        const float v = __fdiv_rn(decode1<FMT>(q[i]), s);
        if (OUT == 0) static_cast<float*>(y)[i] = v;
        else static_cast<uint16_t*>(y)[i] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
    }
}

// MX (1x32 blocks, E8M0 scales) with cols % 32 == 0: a row's blocks are the
// consecutive 32-code runs of the flat array, so group g's block is
// g / (32 / kCodes).  Each CTA owns kThreads x kUnroll consecutive groups.
template <int FMT, int OUT, int OB>
__global__ void __launch_bounds__(kThreads)
k_dequant_mx(const typename DOut<OUT, OB>::In* __restrict__ q, int64_t ngroups, const uint8_t* __restrict__ e8m0,
             typename DOut<OUT, OB>::Out* __restrict__ y) {
    pdl_enter();
    using D = DOut<OUT, OB>;
    constexpr int kGroupsPerBlock = 32 / D::kCodes;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads * kUnroll + threadIdx.x;
    typename D::In c[kUnroll];
    uint32_t b[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t g = base + u * kThreads;
        const bool ok = g < ngroups;
        c[u] = ok ? ld_codes(q + g) : typename D::In{};
        b[u] = ok ? static_cast<uint32_t>(__ldcs(e8m0 + g / kGroupsPerBlock)) : 127u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t g = base + u * kThreads;
        if (g < ngroups) store_words(y + g, D::template multiply<FMT>(c[u], e8m0_to_float(b[u])));
    }
}

// MX over any cols (ragged right edge), element by element.
template <int FMT, int OUT>
__global__ void __launch_bounds__(kThreads)
k_dequant_mx_general(const uint8_t* __restrict__ q, int64_t rows, int64_t cols, const uint8_t* __restrict__ e8m0,
                     void* __restrict__ y) {
    pdl_enter();
    const int64_t n = rows * cols;
    const int64_t nbc = (cols + 31) / 32;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * kThreads) {
        const int64_t r = i / cols, c = i - (i / cols) * cols;
        const float v = __fmul_rn(decode1<FMT>(q[i]), e8m0_to_float(e8m0[r * nbc + c / 32]));
        if (OUT == 0) static_cast<float*>(y)[i] = v;
        else static_cast<uint16_t*>(y)[i] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
    }
}

template <int FMT, int OUT, int OB>
cudaError_t dequant_mx_fast(const uint8_t* q, int64_t n, const uint8_t* e8m0, void* y, cudaStream_t st) {
    using D = DOut<OUT, OB>;
    const int64_t ngroups = n / D::kCodes;  // n is a multiple of 32, so of kCodes
    const int64_t per_cta = static_cast<int64_t>(kThreads) * kUnroll;
    const int64_t grid = std::max<int64_t>(1, (ngroups + per_cta - 1) / per_cta);
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const cudaError_t e = launch_kernel(k_dequant_mx<FMT, OUT, OB>, dim3(static_cast<unsigned>(grid)), dim3(kThreads),
                                        0, st, reinterpret_cast<const typename D::In*>(q), ngroups, e8m0,
                                        static_cast<typename D::Out*>(y));
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int FMT, int OUT>
cudaError_t dequant_mx_typed(const uint8_t* q, int64_t rows, int64_t cols, const uint8_t* e8m0, void* y,
                             cudaStream_t st) {
    const int64_t n = rows * cols;
    if (cols % 32 == 0) {
        if ((reinterpret_cast<uintptr_t>(y) & 31u) == 0) return dequant_mx_fast<FMT, OUT, 32>(q, n, e8m0, y, st);
        return dequant_mx_fast<FMT, OUT, 16>(q, n, e8m0, y, st);
    }
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((n + kThreads - 1) / kThreads,
                                                                static_cast<int64_t>(device_sm_count()) * 8));
    const cudaError_t e = launch_kernel(k_dequant_mx_general<FMT, OUT>, dim3(static_cast<unsigned>(grid)),
                                        dim3(kThreads), 0, st, q, rows, cols, e8m0, y);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int FMT, int OUT, int OB>
cudaError_t dequant_fast(const uint8_t* q, int64_t rows, int64_t cols, int mode, const float* scales, void* y,
                         cudaStream_t st) {
    using D = DOut<OUT, OB>;
    const int64_t n = rows * cols;
    if (mode == 2) {
        const int64_t tiles = ((rows + 127) / 128) * (cols / 128);
        if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
        {
        const cudaError_t e_ = launch_kernel(k_dequant_128x128<FMT, OUT, OB>, dim3(static_cast<unsigned>(tiles)), dim3(kThreads), 0, st, reinterpret_cast<const typename D::In*>(q), scales, static_cast<typename D::Out*>(y), rows, cols);
        if (e_ != cudaSuccess) return e_;
    }
        return cudaGetLastError();
    }
    const int64_t ngroups = n / D::kCodes;
    const int tail_n = static_cast<int>(n - ngroups * D::kCodes);
    const size_t osz = D::kOutElem;
    const int64_t per_cta = static_cast<int64_t>(kThreads) * kUnroll;
    const int64_t grid = std::max<int64_t>(1, (ngroups + per_cta - 1) / per_cta);
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    auto launch = [&](auto kern) -> cudaError_t {
        return launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), 0, st,
                             reinterpret_cast<const typename D::In*>(q), ngroups, q + ngroups * D::kCodes, tail_n,
                             scales, static_cast<typename D::Out*>(y), static_cast<char*>(y) + ngroups * D::kCodes * osz);
    };
    if (mode == 0) return launch(k_dequant_flat<FMT, OUT, OB, 0>);
    return launch(k_dequant_flat<FMT, OUT, OB, 1>);
}

template <int FMT, int OUT>
cudaError_t dequant_typed(const uint8_t* q, int64_t rows, int64_t cols, int mode, const float* scales, void* y,
                          cudaStream_t st) {
    const int64_t n = rows * cols;
    if (mode == 0 || cols % 128 == 0) {
        if ((reinterpret_cast<uintptr_t>(y) & 31u) == 0) return dequant_fast<FMT, OUT, 32>(q, rows, cols, mode, scales, y, st);
        return dequant_fast<FMT, OUT, 16>(q, rows, cols, mode, scales, y, st);
    }
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((n + kThreads - 1) / kThreads,
                                                                static_cast<int64_t>(device_sm_count()) * 8));
    {
        const cudaError_t e_ = launch_kernel(k_dequant_general<FMT, OUT>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), 0, st, q, rows, cols, mode, scales, y);
        if (e_ != cudaSuccess) return e_;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequant_mx(const uint8_t* q, int fmt, int64_t rows, int64_t cols, const uint8_t* e8m0, void* y,
                              int out_dtype, cudaStream_t st) {
    if (fmt == kE4M3) {
        return out_dtype == 0 ? dequant_mx_typed<kE4M3, 0>(q, rows, cols, e8m0, y, st)
                              : dequant_mx_typed<kE4M3, 1>(q, rows, cols, e8m0, y, st);
    }
    return out_dtype == 0 ? dequant_mx_typed<kE5M2, 0>(q, rows, cols, e8m0, y, st)
                          : dequant_mx_typed<kE5M2, 1>(q, rows, cols, e8m0, y, st);
}

cudaError_t launch_dequant(const uint8_t* q, int fmt, int64_t rows, int64_t cols, int mode, const float* scales,
                           void* y, int out_dtype, cudaStream_t st) {
    if (fmt == kE4M3) {
        return out_dtype == 0 ? dequant_typed<kE4M3, 0>(q, rows, cols, mode, scales, y, st)
                              : dequant_typed<kE4M3, 1>(q, rows, cols, mode, scales, y, st);
    }
    return out_dtype == 0 ? dequant_typed<kE5M2, 0>(q, rows, cols, mode, scales, y, st)
                          : dequant_typed<kE5M2, 1>(q, rows, cols, mode, scales, y, st);
}

}  // namespace fp8q
