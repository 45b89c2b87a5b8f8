// fake_quant.cu -- fused FP8 quantize -> dequantize round trip ("fake quant").
//
// PyTorch-FP8 page s3.2 (FP8QuantizeFunction: scale, cast to FP8, cast back)
// and s4.2 DelayedScaler.quantize(); mixed-precision handbook, section "FP8
// training", quant().  In x's own dtype:
//     y = RN_dtype( RN_f32( decode( fp8( RN_f32(x * s) ) ) / s ) )
// with s from each block's amax (1x128, 128x128) or given (per tensor).  One
// pass: x is read once and y written once; the FP8 codes never leave
// registers.  Scales are written only when the caller asks for them.  y may be
// x itself: each lane reads its whole slice before it writes it, and the loads
// here are ordinary coherent loads.

#include <algorithm>

#include "dequant_math.cuh"
#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "launch_util.h"
#include "lane_vec.cuh"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
constexpr int kLoads = 4;

// Coherent (not read-only-path) loads, so that y may alias x.
__device__ __forceinline__ Words<8> ld_words_rw(const Words<8>* p) {
    Words<8> v;
    asm volatile("ld.global.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
                   "=r"(v.w[6]), "=r"(v.w[7])
                 : "l"(p));
    return v;
}
__device__ __forceinline__ Words<4> ld_words_rw(const Words<4>* p) {
    Words<4> v;
    asm volatile("ld.global.L1::no_allocate.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3])
                 : "l"(p));
    return v;
}
__device__ __forceinline__ void st_words(Words<8>* p, const Words<8>& v) {
    V32 o;
#pragma unroll
    for (int k = 0; k < 8; ++k) o.w[k] = v.w[k];
    st32_stream(p, o);
}
__device__ __forceinline__ void st_words(Words<4>* p, const Words<4>& v) {
    st_stream(reinterpret_cast<uint4*>(p), make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]));
}

// The round trip of one lane's slice, element order and width unchanged.
template <typename T, int BYTES, int FMT>
struct RoundTrip;

template <int BYTES, int FMT>
struct RoundTrip<uint16_t, BYTES, FMT> {
    static constexpr int kWords = BYTES / 4;
    using W = Words<kWords>;
    static __device__ __forceinline__ W apply(const W& v, float s) {
        const uint64_t s2 = f32x2(s, s);
        W o;
        if (scale_fast_ok(s)) {
            const float r = __frcp_rn(s);
            const uint64_t r2 = f32x2(r, r);
            const uint64_t ns2 = f32x2(-s, -s);
#pragma unroll
            for (int k = 0; k < kWords; ++k) {
                const float2 y = dequant2_fast<FMT>(scale_cast_bf16x2<FMT>(v.w[k], s2), r2, ns2);
                o.w[k] = pack_bf16x2(y.x, y.y);
            }
        } else {
#pragma unroll
            for (int k = 0; k < kWords; ++k) {
                const float2 y = dequant2_div<FMT>(scale_cast_bf16x2<FMT>(v.w[k], s2), s);
                o.w[k] = pack_bf16x2(y.x, y.y);
            }
        }
        return o;
    }
};

template <int BYTES, int FMT>
struct RoundTrip<float, BYTES, FMT> {
    static constexpr int kWords = BYTES / 4;
    using W = Words<kWords>;
    static __device__ __forceinline__ W apply(const W& v, float s) {
        const uint64_t s2 = f32x2(s, s);
        W o;
        const bool fast = scale_fast_ok(s);
        const float r = __frcp_rn(s);
        const uint64_t r2 = f32x2(r, r);
        const uint64_t ns2 = f32x2(-s, -s);
#pragma unroll
        for (int k = 0; k < kWords; k += 2) {
            const uint32_t c = scale_cast_f32x2<FMT>(v.w[k], v.w[k + 1], s2);
            const float2 y = fast ? dequant2_fast<FMT>(c, r2, ns2) : dequant2_div<FMT>(c, s);
            o.w[k] = __float_as_uint(y.x);
            o.w[k + 1] = __float_as_uint(y.y);
        }
        return o;
    }
};

// 1x128 blocks (cols % 128 == 0): the 1x128 quantizer's one-shot CTA layout.
template <typename T, int FMT, int BYTES>
__global__ void __launch_bounds__(kThreads)
k_fake_quant_1x128(const Words<BYTES / 4>* x, Words<BYTES / 4>* y, float* __restrict__ scales, int64_t nblocks) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    using R = RoundTrip<T, BYTES, FMT>;
    constexpr int kLanesPerBlock = 128 / V::kElems;
    constexpr int kBlocksPerLoad = 32 / kLanesPerBlock;
    const int lane = threadIdx.x & 31;
    const int sub_block = lane / kLanesPerBlock;
    const int64_t nloads = (nblocks + kBlocksPerLoad - 1) / kBlocksPerLoad;
    const int64_t l0 = (static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5)) * kLoads;
    Words<BYTES / 4> v[kLoads];
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
        const int64_t l = l0 + u;
        const int64_t blk = l * kBlocksPerLoad + sub_block;
        v[u] = (l < nloads && blk < nblocks) ? ld_words_rw(x + l * 32 + lane) : V::zero();
    }
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
        const int64_t l = l0 + u;
        const int64_t blk = l * kBlocksPerLoad + sub_block;
        const float s = scale_from_amax<FMT>(warp_max<kLanesPerBlock>(V::amax(v[u])));
        if (l < nloads && blk < nblocks) {
            st_words(y + l * 32 + lane, R::apply(v[u], s));
            if (scales != nullptr && (lane % kLanesPerBlock) == 0) scales[blk] = s;
        }
    }
}

// 128x128 blocks (cols % 128 == 0): register-resident tile, one CTA per tile.
template <typename T, int FMT, int BYTES>
__global__ void __launch_bounds__(kThreads)
k_fake_quant_128x128(const Words<BYTES / 4>* x, Words<BYTES / 4>* y, float* __restrict__ scales, int64_t rows,
                     int64_t cols) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    using R = RoundTrip<T, BYTES, FMT>;
    constexpr int kVecPerRow = 128 / V::kElems;
    constexpr int kRowsPerLoad = 32 / kVecPerRow;
    constexpr int kTileLoads = 16 / kRowsPerLoad;
    __shared__ float warp_amax[kThreads / 32];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t tiles_c = cols >> 7;
    const int64_t tr = blockIdx.x / tiles_c;
    const int64_t tc = blockIdx.x - tr * tiles_c;
    const int64_t vec_cols = cols / V::kElems;
    const int64_t r_base = tr * 128 + warp * 16 + lane / kVecPerRow;
    const int64_t v_base = r_base * vec_cols + tc * kVecPerRow + lane % kVecPerRow;
    Words<BYTES / 4> v[kTileLoads];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kTileLoads; ++i) {
        const int64_t r = r_base + i * kRowsPerLoad;
        v[i] = (r < rows) ? ld_words_rw(x + v_base + i * kRowsPerLoad * vec_cols) : V::zero();
    }
#pragma unroll
    for (int i = 0; i < kTileLoads; ++i) amax = fmaxf(amax, V::amax(v[i]));
    amax = warp_max<32>(amax);
    if (lane == 0) warp_amax[warp] = amax;
    __syncthreads();
    float tile_amax = warp_amax[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) tile_amax = fmaxf(tile_amax, warp_amax[w]);
    const float s = scale_from_amax<FMT>(tile_amax);
#pragma unroll
    for (int i = 0; i < kTileLoads; ++i) {
        const int64_t r = r_base + i * kRowsPerLoad;
        if (r < rows) st_words(y + v_base + i * kRowsPerLoad * vec_cols, R::apply(v[i], s));
    }
    if (scales != nullptr && threadIdx.x == 0) scales[blockIdx.x] = s;
}

template <typename T>
__device__ __forceinline__ float load1(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load1<uint16_t>(const uint16_t* p, int64_t i) {
    return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
}
template <>
__device__ __forceinline__ float load1<float>(const float* p, int64_t i) { return p[i]; }

template <typename T>
__device__ __forceinline__ void store1(T* p, int64_t i, float v);
template <>
__device__ __forceinline__ void store1<uint16_t>(uint16_t* p, int64_t i, float v) {
    p[i] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
}
template <>
__device__ __forceinline__ void store1<float>(float* p, int64_t i, float v) { p[i] = v; }

// One element's round trip with scale s (slow path, any layout).
template <int FMT>
__device__ __forceinline__ float round_trip1(float xv, float s) {
    const uint32_t c = cvt_fp8x2<FMT>(__fmul_rn(xv, s), 0.0f) & 0xFFu;
    return __fdiv_rn(fp8x2_to_float2<FMT>(c).x, s);
}

// Per tensor with a given scale: one-shot chunks of kThreads x kLoads lane
// slices; the tail (< one slice) goes to CTA 0.
template <typename T, int FMT, int BYTES>
__global__ void __launch_bounds__(kThreads)
k_fake_quant_tensor(const Words<BYTES / 4>* x, Words<BYTES / 4>* y, int64_t nvec, const T* x_tail, T* y_tail,
                    int tail_n, const float* scale_in) {
    pdl_enter();
    using R = RoundTrip<T, BYTES, FMT>;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads * kLoads + threadIdx.x;
    Words<BYTES / 4> v[kLoads];
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
        const int64_t i = base + u * kThreads;
        v[u] = (i < nvec) ? ld_words_rw(x + i) : LaneVec<T, BYTES>::zero();
    }
    const float s = *scale_in;
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
        const int64_t i = base + u * kThreads;
        if (i < nvec) st_words(y + i, R::apply(v[u], s));
    }
    if (blockIdx.x == 0 && threadIdx.x < tail_n)
        store1(y_tail, threadIdx.x, round_trip1<FMT>(load1(x_tail, threadIdx.x), s));
}

// Blocks with a ragged right edge (cols % 128 != 0): one CTA per block,
// element by element (amax sweep, then the round trip).
constexpr int kGeneralThreads = 128;

template <typename T, int FMT>
__global__ void __launch_bounds__(kGeneralThreads)
k_fake_quant_general(const T* x, T* y, float* __restrict__ scales, int64_t rows, int64_t cols, int br,
                     int64_t nblocks) {
    pdl_enter();
    __shared__ float warp_amax[kGeneralThreads / 32];
    const int64_t nbc = (cols + 127) / 128;
    for (int64_t b = blockIdx.x; b < nblocks; b += gridDim.x) {
        const int64_t bi = b / nbc, bj = b - (b / nbc) * nbc;
        const int64_t r0 = bi * br, c0 = bj * 128;
        const int64_t h = min(static_cast<int64_t>(br), rows - r0);
        const int64_t w = min(static_cast<int64_t>(128), cols - c0);
        float amax = 0.0f;
        for (int64_t i = threadIdx.x; i < h * w; i += kGeneralThreads)
            amax = fmaxf(amax, fabsf(load1(x, (r0 + i / w) * cols + c0 + i % w)));
        amax = warp_max<32>(amax);
        if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = amax;
        __syncthreads();
        float m = warp_amax[0];
#pragma unroll
        for (int k = 1; k < kGeneralThreads / 32; ++k) m = fmaxf(m, warp_amax[k]);
        __syncthreads();  // every read of x in this block is done before y (which may be x) is written
        const float s = scale_from_amax<FMT>(m);
        for (int64_t i = threadIdx.x; i < h * w; i += kGeneralThreads) {
            const int64_t e = (r0 + i / w) * cols + c0 + i % w;
            store1(y, e, round_trip1<FMT>(load1(x, e), s));
        }
        if (scales != nullptr && threadIdx.x == 0) scales[b] = s;
    }
}

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <typename T, int FMT, int BYTES>
cudaError_t launch_fq_fast(const void* x, void* y, int64_t rows, int64_t cols, int br, const float* scale_in,
                           float* scales, cudaStream_t st) {
    using V = LaneVec<T, BYTES>;
    using W = Words<BYTES / 4>;
    const int64_t n = rows * cols;
    if (br == 0) {
        const int64_t nvec = n / V::kElems;
        const int tail_n = static_cast<int>(n - nvec * V::kElems);
        const int64_t per_cta = static_cast<int64_t>(kThreads) * kLoads;
        const int64_t grid = std::max<int64_t>(1, (nvec + per_cta - 1) / per_cta);
        if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
        {
        const cudaError_t e_ = launch_kernel(k_fake_quant_tensor<T, FMT, BYTES>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), 0, st, static_cast<const W*>(x), static_cast<W*>(y), nvec, static_cast<const T*>(x) + nvec * V::kElems,
            static_cast<T*>(y) + nvec * V::kElems, tail_n, scale_in);
        if (e_ != cudaSuccess) return e_;
    }
    } else if (br == 1) {
        const int64_t nblocks = n / 128;
        constexpr int kBlocksPerLoad = 32 / (128 / V::kElems);
        const int64_t nloads = (nblocks + kBlocksPerLoad - 1) / kBlocksPerLoad;
        const int64_t per_cta = static_cast<int64_t>(kThreads / 32) * kLoads;
        const int64_t grid = (nloads + per_cta - 1) / per_cta;
        if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
        {
        const cudaError_t e_ = launch_kernel(k_fake_quant_1x128<T, FMT, BYTES>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), 0, st, static_cast<const W*>(x), static_cast<W*>(y), scales, nblocks);
        if (e_ != cudaSuccess) return e_;
    }
    } else {
        const int64_t tiles = ((rows + 127) / 128) * (cols / 128);
        if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
        {
        const cudaError_t e_ = launch_kernel(k_fake_quant_128x128<T, FMT, BYTES>, dim3(static_cast<unsigned>(tiles)), dim3(kThreads), 0, st, static_cast<const W*>(x), static_cast<W*>(y), scales, rows, cols);
        if (e_ != cudaSuccess) return e_;
    }
    }
    return cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t launch_fq_typed(const void* x, void* y, int64_t rows, int64_t cols, int br, const float* scale_in,
                            float* scales, cudaStream_t st) {
    if (br == 0 || cols % 128 == 0) {
        if (aligned32(x) && aligned32(y))
            return launch_fq_fast<T, FMT, 32>(x, y, rows, cols, br, scale_in, scales, st);
        return launch_fq_fast<T, FMT, 16>(x, y, rows, cols, br, scale_in, scales, st);
    }
    const int64_t nblocks = ((rows + br - 1) / br) * ((cols + 127) / 128);
    const int64_t grid = std::min<int64_t>(nblocks, static_cast<int64_t>(device_sm_count()) * 16);
    {
        const cudaError_t e_ = launch_kernel(k_fake_quant_general<T, FMT>, dim3(static_cast<unsigned>(grid)), dim3(kGeneralThreads), 0, st, static_cast<const T*>(x), static_cast<T*>(y), scales, rows, cols, br, nblocks);
        if (e_ != cudaSuccess) return e_;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fake_quant(const void* x, int dtype, int64_t rows, int64_t cols, int block_rows, int fmt,
                              const float* scale_in, void* y, float* scales, cudaStream_t st) {
    if (dtype == 1) {
        return fmt == kE4M3 ? launch_fq_typed<uint16_t, kE4M3>(x, y, rows, cols, block_rows, scale_in, scales, st)
                            : launch_fq_typed<uint16_t, kE5M2>(x, y, rows, cols, block_rows, scale_in, scales, st);
    }
    return fmt == kE4M3 ? launch_fq_typed<float, kE4M3>(x, y, rows, cols, block_rows, scale_in, scales, st)
                        : launch_fq_typed<float, kE5M2>(x, y, rows, cols, block_rows, scale_in, scales, st);
}

}  // namespace fp8q
