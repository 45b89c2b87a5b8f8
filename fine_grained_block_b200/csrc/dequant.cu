// dequant.cu -- FP8 dequantization kernels.
//
// PyTorch-FP8 page, s4.1 (divide by the scale to restore the value) and s4.2
// quantize() (.to(dtype) / scale): y = fp32(decode(q) / s), one IEEE
// round-to-nearest division per element, then (bf16 output) one more
// round-to-nearest-even to bf16.
//
// Each thread turns one group of codes into one 16-byte output vector: 8 codes
// for bf16 output, 4 codes for fp32 output.  Consecutive lanes therefore read
// consecutive code groups and write consecutive 16-byte vectors, so both the
// loads and the stores of a warp are contiguous.

#include <algorithm>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

template <int OUT>  // 0 = fp32, 1 = bf16
struct DOut;

template <>
struct DOut<0> {
    static constexpr int kCodes = 4;  // 4 codes -> 16 B of fp32
    using In = uint32_t;
    template <int FMT>
    static __device__ __forceinline__ uint4 convert(In c, float s) {
        const float2 a = fp8x2_to_float2<FMT>(c & 0xFFFFu);
        const float2 b = fp8x2_to_float2<FMT>(c >> 16);
        return make_uint4(__float_as_uint(__fdiv_rn(a.x, s)), __float_as_uint(__fdiv_rn(a.y, s)),
                          __float_as_uint(__fdiv_rn(b.x, s)), __float_as_uint(__fdiv_rn(b.y, s)));
    }
};

template <>
struct DOut<1> {
    static constexpr int kCodes = 8;  // 8 codes -> 16 B of bf16
    using In = uint2;
    template <int FMT>
    static __device__ __forceinline__ uint32_t pair(uint32_t c2, float s) {
        const float2 a = fp8x2_to_float2<FMT>(c2);
        return pack_bf16x2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s));
    }
    template <int FMT>
    static __device__ __forceinline__ uint4 convert(In c, float s) {
        return make_uint4(pair<FMT>(c.x & 0xFFFFu, s), pair<FMT>(c.x >> 16, s),
                          pair<FMT>(c.y & 0xFFFFu, s), pair<FMT>(c.y >> 16, s));
    }
};

__device__ __forceinline__ uint32_t ld_codes(const uint32_t* p) { return __ldcs(reinterpret_cast<const unsigned int*>(p)); }
__device__ __forceinline__ uint2 ld_codes(const uint2* p) { return __ldcs(p); }

// One code -> fp32 (for tails and the general kernel).
template <int FMT>
__device__ __forceinline__ float decode1(uint8_t c) { return fp8x2_to_float2<FMT>(c).x; }

// Per-tensor (MODE 0) and 1x128 (MODE 1, cols % 128 == 0) over a flat range
// of ngroups code groups; a per-tensor tail of < kCodes codes goes to CTA 0.
template <int FMT, int OUT, int MODE>
__global__ void __launch_bounds__(kThreads)
k_dequant_flat(const typename DOut<OUT>::In* __restrict__ q, int64_t ngroups,
               const uint8_t* __restrict__ q_tail, int tail_n, const float* __restrict__ scales,
               uint4* __restrict__ y, void* __restrict__ y_tail) {
    using D = DOut<OUT>;
    constexpr int kGroupsPerBlock = 128 / D::kCodes;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    const float s0 = (MODE == 0) ? scales[0] : 0.0f;
    for (int64_t i0 = tid; i0 < ngroups; i0 += nthreads * kUnroll) {
        typename D::In c[kUnroll];
        float s[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = i0 + u * nthreads;
            const bool ok = g < ngroups;
            c[u] = ok ? ld_codes(q + g) : typename D::In{};
            s[u] = (MODE == 0) ? s0 : (ok ? scales[g / kGroupsPerBlock] : 1.0f);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = i0 + u * nthreads;
            if (g < ngroups) st_stream(y + g, D::template convert<FMT>(c[u], s[u]));
        }
    }
    if (MODE == 0 && blockIdx.x == 0 && threadIdx.x < tail_n) {
        const float v = __fdiv_rn(decode1<FMT>(q_tail[threadIdx.x]), s0);
        if (OUT == 0) static_cast<float*>(y_tail)[threadIdx.x] = v;
        else static_cast<uint16_t*>(y_tail)[threadIdx.x] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
    }
}

// 128x128 (cols % 128 == 0): one CTA per tile, one scale per CTA.  A tile row
// is 128 codes = kGroupsPerRow groups; the CTA sweeps the tile's 128 rows.
template <int FMT, int OUT>
__global__ void __launch_bounds__(kThreads)
k_dequant_128x128(const typename DOut<OUT>::In* __restrict__ q, const float* __restrict__ scales,
                  uint4* __restrict__ y, int64_t rows, int64_t cols) {
    using D = DOut<OUT>;
    constexpr int kGroupsPerRow = 128 / D::kCodes;             // 16 (bf16 out) or 32 (fp32 out)
    constexpr int kRowsPerPass = kThreads / kGroupsPerRow;      // 16 or 8
    constexpr int kPasses = 128 / kRowsPerPass;                 // 8 or 16
    const int64_t tiles_c = cols >> 7;
    const int64_t tr = blockIdx.x / tiles_c;
    const int64_t tc = blockIdx.x - tr * tiles_c;
    const float s = scales[blockIdx.x];
    const int64_t groups_per_tensor_row = cols / D::kCodes;
    const int64_t r0 = tr * 128 + threadIdx.x / kGroupsPerRow;
    const int64_t g0 = r0 * groups_per_tensor_row + tc * kGroupsPerRow + threadIdx.x % kGroupsPerRow;
#pragma unroll
    for (int p0 = 0; p0 < kPasses; p0 += kUnroll) {
        typename D::In c[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t r = r0 + (p0 + u) * kRowsPerPass;
            c[u] = (r < rows) ? ld_codes(q + g0 + (p0 + u) * kRowsPerPass * groups_per_tensor_row) : typename D::In{};
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t r = r0 + (p0 + u) * kRowsPerPass;
            if (r < rows) st_stream(y + g0 + (p0 + u) * kRowsPerPass * groups_per_tensor_row, D::template convert<FMT>(c[u], s));
        }
    }
}

// Any layout, element by element (ragged widths).  mode 1: 1x128, 2: 128x128.
template <int FMT, int OUT>
__global__ void __launch_bounds__(kThreads)
k_dequant_general(const uint8_t* __restrict__ q, int64_t rows, int64_t cols, int mode,
                  const float* __restrict__ scales, void* __restrict__ y) {
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

template <typename Kernel>
int64_t flat_grid(Kernel k, int64_t ngroups) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int64_t full = static_cast<int64_t>(device_sm_count()) * per_sm;
    const int64_t need = (ngroups + static_cast<int64_t>(kThreads) * kUnroll - 1) / (static_cast<int64_t>(kThreads) * kUnroll);
    return std::max<int64_t>(1, std::min(full, need));
}

template <int FMT, int OUT>
cudaError_t dequant_typed(const uint8_t* q, int64_t rows, int64_t cols, int mode, const float* scales, void* y,
                          cudaStream_t st) {
    using D = DOut<OUT>;
    const int64_t n = rows * cols;
    const size_t osz = OUT == 0 ? 4 : 2;
    if (mode == 0 || (mode == 1 && cols % 128 == 0)) {
        const int64_t ngroups = (mode == 0) ? n / D::kCodes : n / D::kCodes;
        const int tail_n = static_cast<int>(n - ngroups * D::kCodes);
        auto launch = [&](auto kern) {
            const int64_t grid = flat_grid(kern, ngroups);
            kern<<<static_cast<unsigned>(grid), kThreads, 0, st>>>(
                reinterpret_cast<const typename D::In*>(q), ngroups, q + ngroups * D::kCodes, tail_n, scales,
                static_cast<uint4*>(y), static_cast<char*>(y) + ngroups * D::kCodes * osz);
        };
        if (mode == 0) launch(k_dequant_flat<FMT, OUT, 0>);
        else launch(k_dequant_flat<FMT, OUT, 1>);
        return cudaGetLastError();
    }
    if (mode == 2 && cols % 128 == 0) {
        const int64_t tiles = ((rows + 127) / 128) * (cols / 128);
        if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
        k_dequant_128x128<FMT, OUT><<<static_cast<unsigned>(tiles), kThreads, 0, st>>>(
            reinterpret_cast<const typename D::In*>(q), scales, static_cast<uint4*>(y), rows, cols);
        return cudaGetLastError();
    }
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((n + kThreads - 1) / kThreads,
                                                                static_cast<int64_t>(device_sm_count()) * 8));
    k_dequant_general<FMT, OUT><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(q, rows, cols, mode, scales, y);
    return cudaGetLastError();
}

}  // namespace

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
