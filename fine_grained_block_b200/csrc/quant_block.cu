// quant_block.cu -- fine-grained (blockwise) FP8 quantization kernels.
//
// Mixed-precision handbook, section "FP8 training", per_block: one scale per
// 1x128 run of an activation row, or per 128x128 tile of a weight.  Each
// kernel does the whole path for its blocks in one pass over x: load, amax,
// scale, scaled cast, code store, scale store.

#include <algorithm>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"

namespace fp8q {
namespace {

constexpr int kThreads = 256;

// Widen one 16-byte vector of T (8 bf16 or 4 fp32) and fold |x| into amax.
template <typename T>
struct Vec16;

template <>
struct Vec16<uint16_t> {  // bf16 bit patterns
    static constexpr int kElems = 8;
    static __device__ __forceinline__ float amax(const uint4& v) {
        uint32_t m = absmax_bf16x2(0u, v.x);
        m = absmax_bf16x2(m, v.y);
        m = absmax_bf16x2(m, v.z);
        m = absmax_bf16x2(m, v.w);
        return bf16x2_hmax(m);
    }
    // 8 codes -> 8 bytes
    template <int FMT>
    static __device__ __forceinline__ uint2 cast(const uint4& v, float s) {
        const uint32_t c0 = cvt_fp8x2<FMT>(__fmul_rn(bf16_lo(v.x), s), __fmul_rn(bf16_hi(v.x), s));
        const uint32_t c1 = cvt_fp8x2<FMT>(__fmul_rn(bf16_lo(v.y), s), __fmul_rn(bf16_hi(v.y), s));
        const uint32_t c2 = cvt_fp8x2<FMT>(__fmul_rn(bf16_lo(v.z), s), __fmul_rn(bf16_hi(v.z), s));
        const uint32_t c3 = cvt_fp8x2<FMT>(__fmul_rn(bf16_lo(v.w), s), __fmul_rn(bf16_hi(v.w), s));
        return make_uint2(c0 | (c1 << 16), c2 | (c3 << 16));
    }
    using Out = uint2;
};

template <>
struct Vec16<float> {
    static constexpr int kElems = 4;
    static __device__ __forceinline__ float amax(const uint4& v) {
        const float a = fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y)));
        const float b = fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)));
        return fmaxf(a, b);
    }
    // 4 codes -> 4 bytes
    template <int FMT>
    static __device__ __forceinline__ uint32_t cast(const uint4& v, float s) {
        const uint32_t c0 = cvt_fp8x2<FMT>(__fmul_rn(__uint_as_float(v.x), s), __fmul_rn(__uint_as_float(v.y), s));
        const uint32_t c1 = cvt_fp8x2<FMT>(__fmul_rn(__uint_as_float(v.z), s), __fmul_rn(__uint_as_float(v.w), s));
        return c0 | (c1 << 16);
    }
    using Out = uint32_t;
};

// ---------------------------------------------------------------------------
// 1x128: a block is 128 consecutive elements.  With 16-byte lanes a block is
// 16 lanes (bf16) or 32 lanes (fp32), so one warp-wide load covers 2 (bf16) or
// 1 (fp32) whole blocks and the block amax is a shuffle reduction inside the
// lane group -- no shared memory, no block barrier.  Each warp takes UNROLL
// consecutive warp-loads per trip (UNROLL * 512 contiguous bytes in flight per
// warp) and the grid strides over the tensor.
// ---------------------------------------------------------------------------
template <typename T, int FMT, int UNROLL>
__global__ void __launch_bounds__(kThreads)
k_quant_1x128(const uint4* __restrict__ x, typename Vec16<T>::Out* __restrict__ q,
              float* __restrict__ scales, int64_t nblocks) {
    using V = Vec16<T>;
    constexpr int kLanesPerBlock = 128 / V::kElems;          // 16 (bf16) or 32 (fp32)
    constexpr int kBlocksPerLoad = 32 / kLanesPerBlock;       // 2 or 1
    const int lane = threadIdx.x & 31;
    const int sub_block = lane / kLanesPerBlock;
    const int64_t nloads = (nblocks + kBlocksPerLoad - 1) / kBlocksPerLoad;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;

    for (int64_t l0 = warp * UNROLL; l0 < nloads; l0 += nwarps * UNROLL) {
        uint4 v[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t l = l0 + u;
            const int64_t blk = l * kBlocksPerLoad + sub_block;
            v[u] = (l < nloads && blk < nblocks) ? ld_stream(x + l * 32 + lane) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t l = l0 + u;
            const int64_t blk = l * kBlocksPerLoad + sub_block;
            const float amax = warp_max<kLanesPerBlock>(V::amax(v[u]));
            const float s = scale_from_amax<FMT>(amax);
            if (l < nloads && blk < nblocks) {
                st_stream(q + l * 32 + lane, V::template cast<FMT>(v[u], s));
                if ((lane % kLanesPerBlock) == 0) scales[blk] = s;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// 128x128: one CTA per tile, 8 warps, each warp owns 16 rows of the tile.  A
// row of the tile is 256 B (bf16) or 512 B (fp32); one warp-wide 16-byte load
// covers 2 rows (bf16) or 1 row (fp32).  The whole tile stays in registers
// (128 B/thread bf16, 256 B/thread fp32) between the amax and the cast, so x
// is read from HBM exactly once.  Tile amax: shuffle within the warp, then
// the 8 warp maxima through shared memory.  Rows past the end (ragged bottom
// edge) are masked; they do not count toward the amax.
// ---------------------------------------------------------------------------
template <typename T, int FMT>
__global__ void __launch_bounds__(kThreads)
k_quant_128x128(const uint4* __restrict__ x, typename Vec16<T>::Out* __restrict__ q,
                float* __restrict__ scales, int64_t rows, int64_t cols) {
    using V = Vec16<T>;
    constexpr int kVecPerRow = 128 / V::kElems;               // 16 (bf16) or 32 (fp32) vectors per tile row
    constexpr int kRowsPerLoad = 32 / kVecPerRow;              // 2 or 1
    constexpr int kLoads = 16 / kRowsPerLoad;                  // 8 or 16 loads per thread
    __shared__ float warp_amax[kThreads / 32];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t tiles_c = cols >> 7;
    const int64_t tr = blockIdx.x / tiles_c;
    const int64_t tc = blockIdx.x - tr * tiles_c;
    const int row_in_load = lane / kVecPerRow;
    const int vec_in_row = lane % kVecPerRow;
    const int64_t vec_cols = cols / V::kElems;                 // 16-byte vectors per tensor row
    const int64_t r_base = tr * 128 + warp * 16 + row_in_load;
    const int64_t v_base = r_base * vec_cols + tc * kVecPerRow + vec_in_row;

    uint4 v[kLoads];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const int64_t r = r_base + i * kRowsPerLoad;
        v[i] = (r < rows) ? ld_stream(x + v_base + i * kRowsPerLoad * vec_cols) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kLoads; ++i) amax = fmaxf(amax, V::amax(v[i]));
    amax = warp_max<32>(amax);
    if (lane == 0) warp_amax[warp] = amax;
    __syncthreads();
    float tile_amax = warp_amax[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) tile_amax = fmaxf(tile_amax, warp_amax[w]);
    const float s = scale_from_amax<FMT>(tile_amax);
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const int64_t r = r_base + i * kRowsPerLoad;
        if (r < rows) st_stream(q + v_base + i * kRowsPerLoad * vec_cols, V::template cast<FMT>(v[i], s));
    }
    if (threadIdx.x == 0) scales[blockIdx.x] = s;
}

// ---------------------------------------------------------------------------
// General blocks: any block shape and any cols (ragged right edge), element
// by element.  One CTA per block; the block is swept twice (amax, then cast),
// the second sweep hitting L1/L2.  Used only when cols % 128 != 0.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float load_elem(const T* x, int64_t i);
template <>
__device__ __forceinline__ float load_elem<uint16_t>(const uint16_t* x, int64_t i) {
    return __uint_as_float(static_cast<uint32_t>(x[i]) << 16);
}
template <>
__device__ __forceinline__ float load_elem<float>(const float* x, int64_t i) { return x[i]; }

constexpr int kGeneralThreads = 128;

template <typename T, int FMT>
__global__ void __launch_bounds__(kGeneralThreads)
k_quant_block_general(const T* __restrict__ x, uint8_t* __restrict__ q, float* __restrict__ scales,
                      int64_t rows, int64_t cols, int br, int bc, int64_t nblocks) {
    __shared__ float warp_amax[kGeneralThreads / 32];
    const int64_t nbc = (cols + bc - 1) / bc;
    for (int64_t b = blockIdx.x; b < nblocks; b += gridDim.x) {
        const int64_t bi = b / nbc, bj = b - (b / nbc) * nbc;
        const int64_t r0 = bi * br, c0 = bj * bc;
        const int64_t h = min(static_cast<int64_t>(br), rows - r0);
        const int64_t w = min(static_cast<int64_t>(bc), cols - c0);
        const int64_t count = h * w;
        float amax = 0.0f;
        for (int64_t i = threadIdx.x; i < count; i += kGeneralThreads) {
            const int64_t r = r0 + i / w, c = c0 + i % w;
            amax = fmaxf(amax, fabsf(load_elem(x, r * cols + c)));
        }
        amax = warp_max<32>(amax);
        if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = amax;
        __syncthreads();
        float blk_amax = warp_amax[0];
#pragma unroll
        for (int k = 1; k < kGeneralThreads / 32; ++k) blk_amax = fmaxf(blk_amax, warp_amax[k]);
        __syncthreads();  // warp_amax is reused by the next block
        const float s = scale_from_amax<FMT>(blk_amax);
        for (int64_t i = threadIdx.x; i < count; i += kGeneralThreads) {
            const int64_t r = r0 + i / w, c = c0 + i % w;
            const float p = __fmul_rn(load_elem(x, r * cols + c), s);
            q[r * cols + c] = static_cast<uint8_t>(cvt_fp8x2<FMT>(p, 0.0f) & 0xFFu);
        }
        if (threadIdx.x == 0) scales[b] = s;
    }
}

template <typename T, int FMT, int UNROLL>
cudaError_t launch_1x128_typed(const void* x, int64_t nblocks, uint8_t* q, float* scales, cudaStream_t st) {
    constexpr int kBlocksPerLoad = (sizeof(T) == 2) ? 2 : 1;
    const int64_t nloads = (nblocks + kBlocksPerLoad - 1) / kBlocksPerLoad;
    const int64_t warps_needed = (nloads + UNROLL - 1) / UNROLL;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quant_1x128<T, FMT, UNROLL>, kThreads, 0);
    if (e != cudaSuccess) return e;
    const int64_t full = static_cast<int64_t>(device_sm_count()) * (per_sm > 0 ? per_sm : 1);
    const int64_t grid = std::min<int64_t>(full, (warps_needed + kThreads / 32 - 1) / (kThreads / 32));
    k_quant_1x128<T, FMT, UNROLL><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(
        static_cast<const uint4*>(x), reinterpret_cast<typename Vec16<T>::Out*>(q), scales, nblocks);
    return cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t launch_128x128_typed(const void* x, int64_t rows, int64_t cols, uint8_t* q, float* scales,
                                 cudaStream_t st) {
    const int64_t tiles = ((rows + 127) / 128) * (cols / 128);
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    k_quant_128x128<T, FMT><<<static_cast<unsigned>(tiles), kThreads, 0, st>>>(
        static_cast<const uint4*>(x), reinterpret_cast<typename Vec16<T>::Out*>(q), scales, rows, cols);
    return cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t launch_general_typed(const void* x, int64_t rows, int64_t cols, int br, int bc, uint8_t* q,
                                 float* scales, cudaStream_t st) {
    const int64_t nblocks = ((rows + br - 1) / br) * ((cols + bc - 1) / bc);
    const int64_t grid = std::min<int64_t>(nblocks, static_cast<int64_t>(device_sm_count()) * 16);
    k_quant_block_general<T, FMT><<<static_cast<unsigned>(grid), kGeneralThreads, 0, st>>>(
        static_cast<const T*>(x), q, scales, rows, cols, br, bc, nblocks);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_1x128(const void* x, int dtype, int64_t nblocks, int fmt, uint8_t* q, float* scales,
                               cudaStream_t st) {
    if (dtype == 1) {
        return fmt == kE4M3 ? launch_1x128_typed<uint16_t, kE4M3, 4>(x, nblocks, q, scales, st)
                            : launch_1x128_typed<uint16_t, kE5M2, 4>(x, nblocks, q, scales, st);
    }
    return fmt == kE4M3 ? launch_1x128_typed<float, kE4M3, 4>(x, nblocks, q, scales, st)
                        : launch_1x128_typed<float, kE5M2, 4>(x, nblocks, q, scales, st);
}

cudaError_t launch_quant_128x128(const void* x, int dtype, int64_t rows, int64_t cols, int fmt, uint8_t* q,
                                 float* scales, cudaStream_t st) {
    if (dtype == 1) {
        return fmt == kE4M3 ? launch_128x128_typed<uint16_t, kE4M3>(x, rows, cols, q, scales, st)
                            : launch_128x128_typed<uint16_t, kE5M2>(x, rows, cols, q, scales, st);
    }
    return fmt == kE4M3 ? launch_128x128_typed<float, kE4M3>(x, rows, cols, q, scales, st)
                        : launch_128x128_typed<float, kE5M2>(x, rows, cols, q, scales, st);
}

cudaError_t launch_quant_block_general(const void* x, int dtype, int64_t rows, int64_t cols, int br, int bc,
                                       int fmt, uint8_t* q, float* scales, cudaStream_t st) {
    if (dtype == 1) {
        return fmt == kE4M3 ? launch_general_typed<uint16_t, kE4M3>(x, rows, cols, br, bc, q, scales, st)
                            : launch_general_typed<uint16_t, kE5M2>(x, rows, cols, br, bc, q, scales, st);
    }
    return fmt == kE4M3 ? launch_general_typed<float, kE4M3>(x, rows, cols, br, bc, q, scales, st)
                        : launch_general_typed<float, kE5M2>(x, rows, cols, br, bc, q, scales, st);
}

}  // namespace fp8q
