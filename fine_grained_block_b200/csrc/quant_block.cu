// quant_block.cu -- fine-grained (blockwise) FP8 quantization kernels.
//
// Mixed-precision handbook, section "FP8 training", per_block: one scale per
// 1x128 run of an activation row, or per 128x128 tile of a weight.  Each
// kernel does the whole path for its blocks in one pass over x: load, amax,
// scale, scaled cast, code store, scale store.

#include <algorithm>
#include <atomic>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "launch_util.h"
#include "lane_vec.cuh"

#ifndef FP8Q_Q128_TMA
#define FP8Q_Q128_TMA 0
#endif
#if FP8Q_Q128_TMA
#include "fp8q_wait.cuh"
#include "tensor_map.h"
#include "umma.cuh"
#endif

namespace fp8q {
namespace {

constexpr int kThreads = 256;

// Warp-loads per warp in the row-block kernel for 1x128 blocks (each CTA covers 8 x LOADS
// warp-loads = 32 KiB of bf16 with 32-byte lanes and LOADS = 4).
#ifndef FP8Q_Q1X128_LOADS
#define FP8Q_Q1X128_LOADS 4
#endif
// The same for the 1x32 MX kernel.
#ifndef FP8Q_QMX_LOADS
#define FP8Q_QMX_LOADS 4
#endif

// Scale rules of the row-block kernel: how a block's amax becomes its scale
// and what is stored for it.
template <int FMT>
struct RatioScale {  // handbook per_block: s = MAX / max(amax, eps), stored as fp32
    using Stored = float;
    static __device__ __forceinline__ float scale(float amax, int, Stored& stored) {
        const float s = scale_from_amax<FMT>(amax);
        stored = s;
        return s;
    }
};
template <int FMT>
struct Pow2Scale {  // MX: s = 2^k, stored as the E8M0 byte of 2^-k
    using Stored = uint8_t;
    static __device__ __forceinline__ float scale(float amax, int rule, Stored& stored) {
        return mx_scale<FMT>(amax, rule, stored);
    }
};

// ---------------------------------------------------------------------------
// Row blocks (1x128, and the 1x32 MX blocks): a block is BW consecutive
// elements.  One lane holds a 16- or 32-byte slice, so a block spans
// BW / kElems lanes (8 lanes for bf16 1x128 with 32-byte slices, 2 for MX) and
// one warp-wide load covers 32 / that many whole blocks.  The block amax is a
// shuffle reduction inside the lane group -- no shared memory, no block
// barrier.  Each CTA owns one contiguous chunk: every warp issues all LOADS of
// its warp-loads before it computes, and finished CTAs are replaced by new
// ones, so each SM keeps its resident CTAs' chunks in flight.
// ---------------------------------------------------------------------------
// One CTA's chunk `cta` of the row blocks (the body of k_quant_rowblocks, also
// run by the grouped kernel for each tensor's chunks).
template <typename T, int FMT, int BYTES, int LOADS, int BW, typename SCALE>
__device__ __forceinline__ void quant_rowblocks_cta(const typename LaneVec<T, BYTES>::In* __restrict__ x,
                                                    typename LaneVec<T, BYTES>::Out* __restrict__ q,
                                                    typename SCALE::Stored* __restrict__ scales, int64_t nblocks,
                                                    int rule, int64_t cta) {
    using V = LaneVec<T, BYTES>;
    constexpr int kLanesPerBlock = BW / V::kElems;
    constexpr int kBlocksPerLoad = 32 / kLanesPerBlock;
    static_assert(kLanesPerBlock >= 1 && kLanesPerBlock <= 32, "a block spans 1..32 lanes");
    const int lane = threadIdx.x & 31;
    const int sub_block = lane / kLanesPerBlock;
    const int64_t nloads = (nblocks + kBlocksPerLoad - 1) / kBlocksPerLoad;
    const int64_t l0 = (cta * (kThreads / 32) + (threadIdx.x >> 5)) * LOADS;

    typename V::In v[LOADS];
#pragma unroll
    for (int u = 0; u < LOADS; ++u) {
        const int64_t l = l0 + u;
        const int64_t blk = l * kBlocksPerLoad + sub_block;
        v[u] = (l < nloads && blk < nblocks) ? ld_words_stream(x + l * 32 + lane) : V::zero();
    }
#pragma unroll
    for (int u = 0; u < LOADS; ++u) {
        const int64_t l = l0 + u;
        const int64_t blk = l * kBlocksPerLoad + sub_block;
        const float amax = warp_max<kLanesPerBlock>(V::amax(v[u]));
        typename SCALE::Stored stored;
        const float s = SCALE::scale(amax, rule, stored);
        if (l < nloads && blk < nblocks) {
            st_stream(q + l * 32 + lane, V::template cast<FMT>(v[u], f32x2(s, s)));
            if ((lane % kLanesPerBlock) == 0) scales[blk] = stored;
        }
    }
}

template <typename T, int FMT, int BYTES, int LOADS, int BW, typename SCALE>
__global__ void __launch_bounds__(kThreads)
k_quant_rowblocks(const typename LaneVec<T, BYTES>::In* __restrict__ x, typename LaneVec<T, BYTES>::Out* __restrict__ q,
                  typename SCALE::Stored* __restrict__ scales, int64_t nblocks, int rule) {
    pdl_enter();
    quant_rowblocks_cta<T, FMT, BYTES, LOADS, BW, SCALE>(x, q, scales, nblocks, rule, blockIdx.x);
}

// ---------------------------------------------------------------------------
// 128x128, register-resident tile: one CTA per tile, 8 warps, each warp owns
// 16 rows of the tile.  One warp-wide load covers 32 / (128 / kElems) tile
// rows.  The whole tile stays in registers between the amax and the cast, so
// x is read from HBM exactly once.  Tile amax: shuffle within the warp, then
// the 8 warp maxima through shared memory.  Rows past the end (ragged bottom
// edge) are masked and do not count toward the amax.  (A TMA-staged tile ring
// was measured against this on B200 and was slower: at 2^28 elements 5461-5520
// GB/s against 6446 GB/s here, because 4 register-resident CTAs per SM keep 4
// tiles both in flight and in process.)
// ---------------------------------------------------------------------------
// Tile `tile` of a [rows, cols] tensor (the body of k_quant_128x128, also run
// by the grouped kernel for each tensor's tiles).
template <typename T, int FMT, int BYTES>
__device__ __forceinline__ void quant_tile_128x128(const typename LaneVec<T, BYTES>::In* __restrict__ x,
                                                   typename LaneVec<T, BYTES>::Out* __restrict__ q,
                                                   float* __restrict__ scales, int64_t rows, int64_t cols,
                                                   int64_t tile) {
    using V = LaneVec<T, BYTES>;
    constexpr int kVecPerRow = 128 / V::kElems;                // lane slices per tile row
    constexpr int kRowsPerLoad = 32 / kVecPerRow;
    constexpr int kLoads = 16 / kRowsPerLoad;                  // loads per thread
    __shared__ float warp_amax[kThreads / 32];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t tiles_c = cols >> 7;
    const int64_t tr = tile / tiles_c;
    const int64_t tc = tile - tr * tiles_c;
    const int row_in_load = lane / kVecPerRow;
    const int vec_in_row = lane % kVecPerRow;
    const int64_t vec_cols = cols / V::kElems;                 // lane slices per tensor row
    const int64_t r_base = tr * 128 + warp * 16 + row_in_load;
    const int64_t v_base = r_base * vec_cols + tc * kVecPerRow + vec_in_row;

    typename V::In v[kLoads];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const int64_t r = r_base + i * kRowsPerLoad;
        v[i] = (r < rows) ? ld_words_stream(x + v_base + i * kRowsPerLoad * vec_cols) : V::zero();
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
    const uint64_t s2 = f32x2(s, s);
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const int64_t r = r_base + i * kRowsPerLoad;
        if (r < rows) st_stream(q + v_base + i * kRowsPerLoad * vec_cols, V::template cast<FMT>(v[i], s2));
    }
    if (threadIdx.x == 0) scales[tile] = s;
}

template <typename T, int FMT, int BYTES>
__global__ void __launch_bounds__(kThreads)
k_quant_128x128(const typename LaneVec<T, BYTES>::In* __restrict__ x, typename LaneVec<T, BYTES>::Out* __restrict__ q,
                float* __restrict__ scales, int64_t rows, int64_t cols) {
    pdl_enter();
    quant_tile_128x128<T, FMT, BYTES>(x, q, scales, rows, cols, blockIdx.x);
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
    pdl_enter();
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

// MX blocks over any cols (ragged right edge): one warp per 1x32 block, lane
// i holding element i of the block; blocks are taken warp-stride.
template <typename T, int FMT>
__global__ void __launch_bounds__(kGeneralThreads)
k_quant_mx_general(const T* __restrict__ x, uint8_t* __restrict__ q, uint8_t* __restrict__ e8m0, int64_t rows,
                   int64_t cols, int64_t nblocks, int rule) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int64_t nbc = (cols + 31) / 32;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (kGeneralThreads / 32);
    for (int64_t b = static_cast<int64_t>(blockIdx.x) * (kGeneralThreads / 32) + (threadIdx.x >> 5); b < nblocks;
         b += warps) {
        const int64_t r = b / nbc, c = (b - r * nbc) * 32 + lane;
        const bool in = c < cols;
        const float v = in ? load_elem(x, r * cols + c) : 0.0f;
        const float amax = warp_max<32>(fabsf(v));
        uint8_t byte;
        const float s = mx_scale<FMT>(amax, rule, byte);
        if (in) q[r * cols + c] = static_cast<uint8_t>(cvt_fp8x2<FMT>(__fmul_rn(v, s), 0.0f) & 0xFFu);
        if (lane == 0) e8m0[b] = byte;
    }
}

// ---------------------------------------------------------------------------
// Grouped: many tensors in one launch.  The tensors' work units (128x128
// tiles, or 1x128 row-block chunks) are numbered consecutively across the
// group; a CTA finds its tensor by binary search over the units' starting
// indices, which travel with the tensors' pointers and shapes in the kernel's
// parameter space.  Many small tensors then cost one launch instead of one
// each, and their blocks fill the GPU together.
// ---------------------------------------------------------------------------
constexpr int kGroupMax = 128;  // tensors per launch (the parameter block stays near 6 KiB)

using GroupEntry = GroupTensor;

struct GroupTable {
    int count;
    int64_t start[kGroupMax + 1];  // start[i] = first unit of tensor i; start[count] = all units
    GroupEntry e[kGroupMax];
};

template <typename T, int FMT, int BYTES, int MODE>
__global__ void __launch_bounds__(kThreads)
k_quant_grouped(const __grid_constant__ GroupTable tab) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    const int64_t b = blockIdx.x;
    int lo = 0, hi = tab.count;  // start[lo] <= b < start[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tab.start[mid] <= b) lo = mid;
        else hi = mid;
    }
    const GroupEntry& e = tab.e[lo];
    const int64_t unit = b - tab.start[lo];
    if (MODE == 2) {
        quant_tile_128x128<T, FMT, BYTES>(static_cast<const typename V::In*>(e.x),
                                          reinterpret_cast<typename V::Out*>(e.q), e.scales, e.rows, e.cols, unit);
    } else {
        quant_rowblocks_cta<T, FMT, BYTES, FP8Q_Q1X128_LOADS, 128, RatioScale<FMT>>(
            static_cast<const typename V::In*>(e.x), reinterpret_cast<typename V::Out*>(e.q), e.scales,
            e.rows * e.cols / 128, 0, unit);
    }
}

template <typename T, int FMT, int BYTES, int LOADS, int BW, typename SCALE>
cudaError_t launch_rowblocks_typed(const void* x, int64_t nblocks, uint8_t* q, typename SCALE::Stored* scales,
                                   int rule, cudaStream_t st) {
    using V = LaneVec<T, BYTES>;
    constexpr int kBlocksPerLoad = 32 / (BW / V::kElems);
    const int64_t nloads = (nblocks + kBlocksPerLoad - 1) / kBlocksPerLoad;
    const int64_t per_cta = static_cast<int64_t>(kThreads / 32) * LOADS;
    const int64_t grid = (nloads + per_cta - 1) / per_cta;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const cudaError_t e = launch_kernel(k_quant_rowblocks<T, FMT, BYTES, LOADS, BW, SCALE>,
                                        dim3(static_cast<unsigned>(grid)), dim3(kThreads), 0, st,
                                        static_cast<const typename V::In*>(x), reinterpret_cast<typename V::Out*>(q),
                                        scales, nblocks, rule);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename T, int FMT, int BYTES, int LOADS>
cudaError_t launch_1x128_typed(const void* x, int64_t nblocks, uint8_t* q, float* scales, cudaStream_t st) {
    return launch_rowblocks_typed<T, FMT, BYTES, LOADS, 128, RatioScale<FMT>>(x, nblocks, q, scales, 0, st);
}

template <typename T, int FMT, int BYTES>
cudaError_t launch_mx_typed(const void* x, int64_t nblocks, uint8_t* q, uint8_t* e8m0, int rule, cudaStream_t st) {
    return launch_rowblocks_typed<T, FMT, BYTES, FP8Q_QMX_LOADS, 32, Pow2Scale<FMT>>(x, nblocks, q, e8m0, rule, st);
}

template <typename T, int FMT, int BYTES>
cudaError_t launch_128x128_typed(const void* x, int64_t rows, int64_t cols, uint8_t* q, float* scales,
                                 cudaStream_t st) {
    using V = LaneVec<T, BYTES>;
    const int64_t tiles = ((rows + 127) / 128) * (cols / 128);
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    {
        const cudaError_t e_ = launch_kernel(k_quant_128x128<T, FMT, BYTES>, dim3(static_cast<unsigned>(tiles)), dim3(kThreads), 0, st, static_cast<const typename V::In*>(x), reinterpret_cast<typename V::Out*>(q), scales, rows, cols);
        if (e_ != cudaSuccess) return e_;
    }
    return cudaGetLastError();
}

#if FP8Q_Q128_TMA
// ---------------------------------------------------------------------------
// A TMA-staged variant of the 128x128 kernel, compiled in only with
// -DFP8Q_Q128_TMA=1 (bf16, rows and cols multiples of 128).  It exists to
// measure the alternative the default kernel was chosen over: persistent
// CTAs keep FP8Q_Q128_TMA_STAGES tiles in flight per CTA, each brought into
// shared memory by one 2-D TMA load (no multicast) on an mbarrier; the tile is
// read into registers, its amax reduced (one barrier per tile), the stage
// reissued for the tile kStages ahead, and the codes cast from registers.
// ---------------------------------------------------------------------------
#ifndef FP8Q_Q128_TMA_STAGES
#define FP8Q_Q128_TMA_STAGES 2
#endif
#ifndef FP8Q_Q128_TMA_CTAS
#define FP8Q_Q128_TMA_CTAS 3
#endif
constexpr int kQtStages = FP8Q_Q128_TMA_STAGES;
constexpr int kQtTileBytes = 128 * 128 * 2;
constexpr int kQtAlloc = kQtStages * kQtTileBytes + 2 * 8 * 4 + kQtStages * 8 + 128;

template <int FMT>
__global__ void __launch_bounds__(kThreads, FP8Q_Q128_TMA_CTAS)
k_quant_128x128_tma(const __grid_constant__ CUtensorMap map_x, uint4* __restrict__ q, float* __restrict__ scales,
                    int64_t rows, int64_t cols, unsigned int* status) {
    using V = LaneVec<uint16_t, 32>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    float (*warp_amax)[8] = reinterpret_cast<float (*)[8]>(sm + kQtStages * kQtTileBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kQtStages * kQtTileBytes + 2 * 8 * 4);
    const int64_t tiles_c = cols / 128, tiles = (rows / 128) * tiles_c;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lr0 = warp * 16 + lane / 8, vec_in_row = lane % 8;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQtStages; ++s) umma::mbar_init(&full[s], 1);
        umma::fence_mbar_init();
    }
    __syncthreads();
    pdl_enter();
    auto issue = [&](int64_t t, int s) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        umma::mbar_arrive_expect_tx(&full[s], kQtTileBytes);
        umma::tma_load_2d(sm + s * kQtTileBytes, &map_x, &full[s], static_cast<int>(tc * 128),
                          static_cast<int>(tr * 128));
    };
    if (threadIdx.x == 0)
        for (int s = 0; s < kQtStages; ++s) {
            const int64_t t = blockIdx.x + static_cast<int64_t>(s) * gridDim.x;
            if (t < tiles) issue(t, s);
        }
    bool timed_out = false;
    int i = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int s = i % kQtStages;
        const bool ok = umma::mbar_wait(&full[s], static_cast<uint32_t>(i / kQtStages) & 1u, kWaitLimitNs);
        const uint8_t* stage = sm + s * kQtTileBytes;
        typename V::In v[4];
        float a = 0.0f;
        if (ok) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint8_t* p = stage + (lr0 + 4 * k) * 256 + vec_in_row * 32;
                const uint4 lo = *reinterpret_cast<const uint4*>(p), hi = *reinterpret_cast<const uint4*>(p + 16);
                v[k] = typename V::In{{lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w}};
                a = fmaxf(a, V::amax(v[k]));
            }
        }
        a = warp_max<32>(a);
        if (lane == 0) warp_amax[i & 1][warp] = a;
        if (__syncthreads_or(!ok)) {
            timed_out = true;
            break;
        }
        if (threadIdx.x == 0) {  // every thread holds its slice: the stage is free
            const int64_t tn = t + static_cast<int64_t>(kQtStages) * gridDim.x;
            if (tn < tiles) issue(tn, s);
        }
        float ta = warp_amax[i & 1][0];
#pragma unroll
        for (int w = 1; w < 8; ++w) ta = fmaxf(ta, warp_amax[i & 1][w]);
        const float sc = scale_from_amax<FMT>(ta);
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            st_stream(q + ((tr * 128 + lr0 + 4 * k) * cols + tc * 128) / 16 + vec_in_row,
                      V::template cast<FMT>(v[k], f32x2(sc, sc)));
        if (threadIdx.x == 0) scales[t] = sc;
    }
    if (timed_out) {
        if (threadIdx.x == 0) {
            atomicOr(status, kStatusWaitTimeout);
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 1000000ull) {
            }
        }
        __syncthreads();
    }
}

template <int FMT>
cudaError_t launch_128x128_tma(const void* x, int64_t rows, int64_t cols, uint8_t* q, float* scales, cudaStream_t st,
                               bool* launched) {
    *launched = false;
    if (rows % 128 != 0 || rows > 0x7FFFFFFF || cols > 0x7FFFFFFF) return cudaSuccess;
    CUtensorMap map;
    if (!make_bf16_tile_map(&map, x, rows, cols, 128, 128)) return cudaSuccess;
    unsigned int* status = device_status_word();
    if (status == nullptr) return cudaSuccess;
    auto kern = k_quant_128x128_tma<FMT>;
    static std::atomic<int> resident[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
    int units = resident[dev].load(std::memory_order_acquire);
    if (units <= 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQtAlloc);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, kQtAlloc);
        if (e != cudaSuccess) return e;
        units = std::max(1, per_sm) * device_sm_count();
        resident[dev].store(units, std::memory_order_release);
    }
    const int64_t grid = std::min<int64_t>((rows / 128) * (cols / 128), units);
    const cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kQtAlloc, st, map,
                                        reinterpret_cast<uint4*>(q), scales, rows, cols, status);
    if (e == cudaSuccess) *launched = true;
    return e;
}
#endif  // FP8Q_Q128_TMA

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <typename T, int FMT>
cudaError_t launch_general_typed(const void* x, int64_t rows, int64_t cols, int br, int bc, uint8_t* q,
                                 float* scales, cudaStream_t st) {
    const int64_t nblocks = ((rows + br - 1) / br) * ((cols + bc - 1) / bc);
    const int64_t grid = std::min<int64_t>(nblocks, static_cast<int64_t>(device_sm_count()) * 16);
    {
        const cudaError_t e_ = launch_kernel(k_quant_block_general<T, FMT>, dim3(static_cast<unsigned>(grid)), dim3(kGeneralThreads), 0, st, static_cast<const T*>(x), q, scales, rows, cols, br, bc, nblocks);
        if (e_ != cudaSuccess) return e_;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_1x128(const void* x, int dtype, int64_t nblocks, int fmt, uint8_t* q, float* scales,
                               cudaStream_t st) {
    const bool w32 = aligned32(x);
    if (dtype == 1) {
        if (w32)
            return fmt == kE4M3 ? launch_1x128_typed<uint16_t, kE4M3, 32, FP8Q_Q1X128_LOADS>(x, nblocks, q, scales, st)
                                : launch_1x128_typed<uint16_t, kE5M2, 32, FP8Q_Q1X128_LOADS>(x, nblocks, q, scales, st);
        return fmt == kE4M3 ? launch_1x128_typed<uint16_t, kE4M3, 16, FP8Q_Q1X128_LOADS>(x, nblocks, q, scales, st)
                            : launch_1x128_typed<uint16_t, kE5M2, 16, FP8Q_Q1X128_LOADS>(x, nblocks, q, scales, st);
    }
    if (w32)
        return fmt == kE4M3 ? launch_1x128_typed<float, kE4M3, 32, FP8Q_Q1X128_LOADS>(x, nblocks, q, scales, st)
                            : launch_1x128_typed<float, kE5M2, 32, FP8Q_Q1X128_LOADS>(x, nblocks, q, scales, st);
    return fmt == kE4M3 ? launch_1x128_typed<float, kE4M3, 16, FP8Q_Q1X128_LOADS>(x, nblocks, q, scales, st)
                        : launch_1x128_typed<float, kE5M2, 16, FP8Q_Q1X128_LOADS>(x, nblocks, q, scales, st);
}

cudaError_t launch_quant_128x128(const void* x, int dtype, int64_t rows, int64_t cols, int fmt, uint8_t* q,
                                 float* scales, cudaStream_t st) {
#if FP8Q_Q128_TMA
    if (dtype == 1) {
        bool launched = false;
        const cudaError_t e = fmt == kE4M3 ? launch_128x128_tma<kE4M3>(x, rows, cols, q, scales, st, &launched)
                                           : launch_128x128_tma<kE5M2>(x, rows, cols, q, scales, st, &launched);
        if (e != cudaSuccess || launched) return e;
    }
#endif
    const bool w32 = aligned32(x);
    if (dtype == 1) {
        if (w32)
            return fmt == kE4M3 ? launch_128x128_typed<uint16_t, kE4M3, 32>(x, rows, cols, q, scales, st)
                                : launch_128x128_typed<uint16_t, kE5M2, 32>(x, rows, cols, q, scales, st);
        return fmt == kE4M3 ? launch_128x128_typed<uint16_t, kE4M3, 16>(x, rows, cols, q, scales, st)
                            : launch_128x128_typed<uint16_t, kE5M2, 16>(x, rows, cols, q, scales, st);
    }
    if (w32)
        return fmt == kE4M3 ? launch_128x128_typed<float, kE4M3, 32>(x, rows, cols, q, scales, st)
                            : launch_128x128_typed<float, kE5M2, 32>(x, rows, cols, q, scales, st);
    return fmt == kE4M3 ? launch_128x128_typed<float, kE4M3, 16>(x, rows, cols, q, scales, st)
                        : launch_128x128_typed<float, kE5M2, 16>(x, rows, cols, q, scales, st);
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

namespace {

// Work units of one tensor in the grouped kernel.
template <typename T, int BYTES>
int64_t group_units(int64_t rows, int64_t cols, int block_rows) {
    if (rows == 0 || cols == 0) return 0;
    if (block_rows == 128) return ((rows + 127) / 128) * (cols / 128);
    using V = LaneVec<T, BYTES>;
    constexpr int kBlocksPerLoad = 32 / (128 / V::kElems);
    const int64_t nblocks = rows * cols / 128;
    const int64_t nloads = (nblocks + kBlocksPerLoad - 1) / kBlocksPerLoad;
    const int64_t per_cta = static_cast<int64_t>(kThreads / 32) * FP8Q_Q1X128_LOADS;
    return (nloads + per_cta - 1) / per_cta;
}

template <typename T, int FMT, int BYTES>
cudaError_t launch_grouped_typed(const GroupTensor* t, int count, int block_rows, cudaStream_t st) {
    GroupTable tab;
    for (int first = 0; first < count; first += kGroupMax) {
        tab.count = std::min(kGroupMax, count - first);
        int64_t units = 0;
        for (int i = 0; i < tab.count; ++i) {
            tab.e[i] = t[first + i];
            tab.start[i] = units;
            units += group_units<T, BYTES>(t[first + i].rows, t[first + i].cols, block_rows);
        }
        tab.start[tab.count] = units;
        if (units == 0) continue;
        if (units > 0x7FFFFFFF) return cudaErrorInvalidValue;
        auto kern = block_rows == 128 ? k_quant_grouped<T, FMT, BYTES, 2> : k_quant_grouped<T, FMT, BYTES, 1>;
        const cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(units)), dim3(kThreads), 0, st, tab);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t launch_grouped_width(const GroupTensor* t, int count, int block_rows, cudaStream_t st) {
    bool w32 = true;  // 256-bit lanes only when every tensor allows them
    for (int i = 0; i < count; ++i) w32 = w32 && aligned32(t[i].x);
    return w32 ? launch_grouped_typed<T, FMT, 32>(t, count, block_rows, st)
               : launch_grouped_typed<T, FMT, 16>(t, count, block_rows, st);
}

}  // namespace

cudaError_t launch_quant_grouped(const GroupTensor* t, int count, int dtype, int block_rows, int fmt,
                                 cudaStream_t st) {
    if (dtype == 1)
        return fmt == kE4M3 ? launch_grouped_width<uint16_t, kE4M3>(t, count, block_rows, st)
                            : launch_grouped_width<uint16_t, kE5M2>(t, count, block_rows, st);
    return fmt == kE4M3 ? launch_grouped_width<float, kE4M3>(t, count, block_rows, st)
                        : launch_grouped_width<float, kE5M2>(t, count, block_rows, st);
}

cudaError_t launch_quant_mx(const void* x, int dtype, int64_t rows, int64_t cols, int fmt, int rule, uint8_t* q,
                            uint8_t* e8m0, cudaStream_t st) {
    if (cols % 32 != 0) {
        const int64_t nblocks = rows * ((cols + 31) / 32);
        const int64_t grid = std::max<int64_t>(
            1, std::min<int64_t>((nblocks + kGeneralThreads / 32 - 1) / (kGeneralThreads / 32),
                                 static_cast<int64_t>(device_sm_count()) * 16));
        auto go = [&](auto kern, auto* xt) -> cudaError_t {
            const cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kGeneralThreads), 0, st,
                                                xt, q, e8m0, rows, cols, nblocks, rule);
            return e != cudaSuccess ? e : cudaGetLastError();
        };
        if (dtype == 1) {
            const auto* xt = static_cast<const uint16_t*>(x);
            return fmt == kE4M3 ? go(k_quant_mx_general<uint16_t, kE4M3>, xt) : go(k_quant_mx_general<uint16_t, kE5M2>, xt);
        }
        const auto* xt = static_cast<const float*>(x);
        return fmt == kE4M3 ? go(k_quant_mx_general<float, kE4M3>, xt) : go(k_quant_mx_general<float, kE5M2>, xt);
    }
    const int64_t nblocks = rows * (cols / 32);
    const bool w32 = aligned32(x);
    if (dtype == 1) {
        if (w32)
            return fmt == kE4M3 ? launch_mx_typed<uint16_t, kE4M3, 32>(x, nblocks, q, e8m0, rule, st)
                                : launch_mx_typed<uint16_t, kE5M2, 32>(x, nblocks, q, e8m0, rule, st);
        return fmt == kE4M3 ? launch_mx_typed<uint16_t, kE4M3, 16>(x, nblocks, q, e8m0, rule, st)
                            : launch_mx_typed<uint16_t, kE5M2, 16>(x, nblocks, q, e8m0, rule, st);
    }
    if (w32)
        return fmt == kE4M3 ? launch_mx_typed<float, kE4M3, 32>(x, nblocks, q, e8m0, rule, st)
                            : launch_mx_typed<float, kE5M2, 32>(x, nblocks, q, e8m0, rule, st);
    return fmt == kE4M3 ? launch_mx_typed<float, kE4M3, 16>(x, nblocks, q, e8m0, rule, st)
                        : launch_mx_typed<float, kE5M2, 16>(x, nblocks, q, e8m0, rule, st);
}

}  // namespace fp8q
