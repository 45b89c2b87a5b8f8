// quant_tensor.cu -- per-tensor FP8 quantization kernels.
//
// Mixed-precision handbook, section "FP8 training", per_tensor: one scale for
// the whole tensor.  PyTorch-FP8 page s4.1 (scale = max_val / amax) and s4.2
// (delayed scaling: the scale comes from earlier steps' amax, so the cast
// needs no global reduction first).
//
// Current scaling is two grid-wide passes: k_tensor_amax (one atomicMax per
// CTA into the caller's amax_out), then k_tensor_cast, which turns that amax
// into s in every CTA.  The cast pass walks the tensor in the reverse order of
// the amax pass, so its first reads find the most recently read data still in
// L2.  Delayed scaling is one pass: cast with the given s and reduce this
// step's amax from the same registers.

#include <algorithm>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

template <typename T>
struct TVec;

template <>
struct TVec<uint16_t> {  // bf16
    static constexpr int kElems = 8;
    using Out = uint2;
    static __device__ __forceinline__ float amax(const uint4& v) {
        uint32_t m = absmax_bf16x2(0u, v.x);
        m = absmax_bf16x2(m, v.y);
        m = absmax_bf16x2(m, v.z);
        m = absmax_bf16x2(m, v.w);
        return bf16x2_hmax(m);
    }
    template <int FMT>
    static __device__ __forceinline__ Out cast(const uint4& v, float s) {
        const uint32_t c0 = cvt_fp8x2<FMT>(__fmul_rn(bf16_lo(v.x), s), __fmul_rn(bf16_hi(v.x), s));
        const uint32_t c1 = cvt_fp8x2<FMT>(__fmul_rn(bf16_lo(v.y), s), __fmul_rn(bf16_hi(v.y), s));
        const uint32_t c2 = cvt_fp8x2<FMT>(__fmul_rn(bf16_lo(v.z), s), __fmul_rn(bf16_hi(v.z), s));
        const uint32_t c3 = cvt_fp8x2<FMT>(__fmul_rn(bf16_lo(v.w), s), __fmul_rn(bf16_hi(v.w), s));
        return make_uint2(c0 | (c1 << 16), c2 | (c3 << 16));
    }
    static __device__ __forceinline__ float elem(const uint16_t* p, int64_t i) {
        return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
    }
};

template <>
struct TVec<float> {
    static constexpr int kElems = 4;
    using Out = uint32_t;
    static __device__ __forceinline__ float amax(const uint4& v) {
        const float a = fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y)));
        const float b = fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)));
        return fmaxf(a, b);
    }
    template <int FMT>
    static __device__ __forceinline__ Out cast(const uint4& v, float s) {
        const uint32_t c0 = cvt_fp8x2<FMT>(__fmul_rn(__uint_as_float(v.x), s), __fmul_rn(__uint_as_float(v.y), s));
        const uint32_t c1 = cvt_fp8x2<FMT>(__fmul_rn(__uint_as_float(v.z), s), __fmul_rn(__uint_as_float(v.w), s));
        return c0 | (c1 << 16);
    }
    static __device__ __forceinline__ float elem(const float* p, int64_t i) { return p[i]; }
};

// CTA-wide max, then one atomicMax per CTA.
__device__ __forceinline__ void cta_amax_to_global(float a, float* amax_out) {
    __shared__ float warp_amax[kThreads / 32];
    a = warp_max<32>(a);
    if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = warp_amax[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, warp_amax[w]);
        atomic_max_nonneg(amax_out, m);
    }
}

// Pass 1 of current scaling.  x is nvec 16-byte vectors followed by tail_n
// (< one vector) trailing elements, which CTA 0 takes.
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_tensor_amax(const uint4* __restrict__ x, int64_t nvec, const T* __restrict__ tail, int tail_n,
              float* __restrict__ amax_out) {
    using V = TVec<T>;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    float a = 0.0f;
    for (int64_t i0 = tid; i0 < nvec; i0 += nthreads * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + u * nthreads;
            v[u] = (i < nvec) ? x[i] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) a = fmaxf(a, V::amax(v[u]));
    }
    if (blockIdx.x == 0 && threadIdx.x < tail_n) a = fmaxf(a, fabsf(V::elem(tail, threadIdx.x)));
    cta_amax_to_global(a, amax_out);
}

// Pass 2 of current scaling (DELAYED = false: s from *amax_in), or the single
// pass of delayed scaling (DELAYED = true: s = *scale_in; WITH_AMAX also
// reduces amax(x) into *amax_out).  Vectors are visited last-to-first.
template <typename T, int FMT, bool DELAYED, bool WITH_AMAX>
__global__ void __launch_bounds__(kThreads)
k_tensor_cast(const uint4* __restrict__ x, int64_t nvec, const T* __restrict__ tail, int tail_n,
              const float* scale_in, const float* __restrict__ amax_in,
              typename TVec<T>::Out* __restrict__ q, uint8_t* __restrict__ q_tail,
              float* scale_out, float* __restrict__ amax_out) {
    using V = TVec<T>;
    const float s = DELAYED ? *scale_in : scale_from_amax<FMT>(*amax_in);
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    float a = 0.0f;
    for (int64_t i0 = tid; i0 < nvec; i0 += nthreads * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + u * nthreads;
            v[u] = (i < nvec) ? ld_stream(x + (nvec - 1 - i)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + u * nthreads;
            if (WITH_AMAX) a = fmaxf(a, V::amax(v[u]));
            if (i < nvec) st_stream(q + (nvec - 1 - i), V::template cast<FMT>(v[u], s));
        }
    }
    if (blockIdx.x == 0 && threadIdx.x < tail_n) {
        const float xv = V::elem(tail, threadIdx.x);
        if (WITH_AMAX) a = fmaxf(a, fabsf(xv));
        q_tail[threadIdx.x] = static_cast<uint8_t>(cvt_fp8x2<FMT>(__fmul_rn(xv, s), 0.0f) & 0xFFu);
    }
    if (WITH_AMAX) cta_amax_to_global(a, amax_out);
    // Written after every read of *scale_in in this CTA (the caller may pass
    // the same pointer for both; other CTAs read the same value either way).
    if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = s;
}

template <typename Kernel>
int64_t grid_for(Kernel k, int64_t nvec) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int64_t full = static_cast<int64_t>(device_sm_count()) * per_sm;
    const int64_t need = (nvec + static_cast<int64_t>(kThreads) * kUnroll - 1) / (static_cast<int64_t>(kThreads) * kUnroll);
    return std::max<int64_t>(1, std::min(full, need));
}

template <typename T>
cudaError_t amax_typed(const void* x, int64_t n, float* amax_out, cudaStream_t st) {
    constexpr int E = TVec<T>::kElems;
    const int64_t nvec = n / E;
    const int tail_n = static_cast<int>(n - nvec * E);
    const T* tail = static_cast<const T*>(x) + nvec * E;
    const int64_t grid = grid_for(k_tensor_amax<T>, nvec);
    k_tensor_amax<T><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(static_cast<const uint4*>(x), nvec, tail,
                                                                     tail_n, amax_out);
    return cudaGetLastError();
}

template <typename T, int FMT, bool DELAYED, bool WITH_AMAX>
cudaError_t cast_typed(const void* x, int64_t n, const float* scale_in, const float* amax_in, uint8_t* q,
                       float* scale_out, float* amax_out, cudaStream_t st) {
    constexpr int E = TVec<T>::kElems;
    const int64_t nvec = n / E;
    const int tail_n = static_cast<int>(n - nvec * E);
    const T* tail = static_cast<const T*>(x) + nvec * E;
    auto kern = k_tensor_cast<T, FMT, DELAYED, WITH_AMAX>;
    const int64_t grid = grid_for(kern, nvec);
    kern<<<static_cast<unsigned>(grid), kThreads, 0, st>>>(
        static_cast<const uint4*>(x), nvec, tail, tail_n, scale_in, amax_in,
        reinterpret_cast<typename TVec<T>::Out*>(q), q + nvec * E, scale_out, amax_out);
    return cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t cast_dispatch(const void* x, int64_t n, const float* scale_in, const float* amax_in, uint8_t* q,
                          float* scale_out, float* amax_out, cudaStream_t st) {
    if (scale_in == nullptr) return cast_typed<T, FMT, false, false>(x, n, nullptr, amax_in, q, scale_out, nullptr, st);
    if (amax_out != nullptr) return cast_typed<T, FMT, true, true>(x, n, scale_in, nullptr, q, scale_out, amax_out, st);
    return cast_typed<T, FMT, true, false>(x, n, scale_in, nullptr, q, scale_out, nullptr, st);
}

}  // namespace

cudaError_t launch_tensor_amax(const void* x, int dtype, int64_t n, float* amax_out, cudaStream_t st) {
    return dtype == 1 ? amax_typed<uint16_t>(x, n, amax_out, st) : amax_typed<float>(x, n, amax_out, st);
}

cudaError_t launch_tensor_cast(const void* x, int dtype, int64_t n, int fmt, const float* scale_in,
                               const float* amax_in, uint8_t* q, float* scale_out, float* amax_out,
                               cudaStream_t st) {
    if (dtype == 1) {
        return fmt == kE4M3 ? cast_dispatch<uint16_t, kE4M3>(x, n, scale_in, amax_in, q, scale_out, amax_out, st)
                            : cast_dispatch<uint16_t, kE5M2>(x, n, scale_in, amax_in, q, scale_out, amax_out, st);
    }
    return fmt == kE4M3 ? cast_dispatch<float, kE4M3>(x, n, scale_in, amax_in, q, scale_out, amax_out, st)
                        : cast_dispatch<float, kE5M2>(x, n, scale_in, amax_in, q, scale_out, amax_out, st);
}

}  // namespace fp8q
