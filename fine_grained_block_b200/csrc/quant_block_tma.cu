// quant_block_tma.cu -- 128x128 block quantization with TMA-staged tiles.
//
// Mixed-precision handbook, section "FP8 training", per_block with 128x128
// blocks (the weight layout): one scale per 128x128 tile.
//
// Persistent CTAs, two per SM.  Each CTA owns tiles blockIdx.x, +gridDim.x,
// ... and keeps STAGES of them in flight in a shared-memory ring: thread 0
// issues one 2-D tensor copy (cp.async.bulk.tensor, no multicast) per tile,
// completing on that stage's mbarrier.  All 8 warps then read the tile from
// shared memory into registers (16 rows per warp, 16 B per lane), reduce the
// tile amax (shuffles, then the 8 warp maxima through shared memory), and
// thread 0 refills the freed stage with the tile STAGES ahead while the warps
// scale, cast and store the codes.  x is read from HBM once; rows beyond the
// tensor (ragged bottom edge) arrive as zeros from the copy engine and are not
// stored.

#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "fp8q_tma.cuh"
#include "lane_vec.cuh"

namespace fp8q {

namespace {

constexpr int kTmaThreads = 256;
constexpr int kTileBytes = 128 * 128 * 2;  // one bf16 tile
#ifndef FP8Q_TMA_STAGES
#define FP8Q_TMA_STAGES 3
#endif
#ifndef FP8Q_TMA_CTAS
#define FP8Q_TMA_CTAS 2
#endif
constexpr int kStages = FP8Q_TMA_STAGES;   // tiles in flight per CTA
constexpr int kCtasPerSm = FP8Q_TMA_CTAS;  // independent pipelines per SM

using TileVec = LaneVec<uint16_t, 16>;  // 16 bytes of a tile row per lane

template <int FMT, int STAGES>
__global__ void __launch_bounds__(kTmaThreads, kCtasPerSm)
k_quant_128x128_tma(const __grid_constant__ CUtensorMap tmap, uint2* __restrict__ q, float* __restrict__ scales,
                    int64_t rows, int64_t cols, int64_t ntiles, unsigned int* status) {
    extern __shared__ uint8_t smem_raw[];
    // tiles first (128-byte aligned for the copy engine), then the barriers
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t* full = reinterpret_cast<uint64_t*>(tiles + STAGES * kTileBytes);
    __shared__ float red[2][kTmaThreads / 32];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t tiles_c = cols >> 7;
    const int64_t grid = gridDim.x;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](int stage, int64_t t) {
        const int64_t tr = t / tiles_c;
        const int64_t tc = t - tr * tiles_c;
        mbar_arrive_expect_tx(&full[stage], kTileBytes);
        tma_load_2d(tiles + stage * kTileBytes, &tmap, &full[stage], static_cast<int>(tc * 128),
                    static_cast<int>(tr * 128));
    };
    int64_t issued = 0;  // tiles issued by this CTA (thread 0's count)
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            const int64_t t = blockIdx.x + s * grid;
            if (t < ntiles) {
                issue(s, t);
                ++issued;
            }
        }
    }

    const int row_in_load = lane >> 4;  // a warp-wide 16-byte access covers 2 tile rows
    const int chunk = lane & 15;        // 16-byte chunk within the 256-byte tile row
    const int64_t q_cols = cols >> 3;   // uint2 (8 codes) per tensor row
    int64_t i = 0;
    for (;; ++i) {
        const int64_t t = blockIdx.x + i * grid;
        if (t >= ntiles) break;
        const int stage = static_cast<int>(i % STAGES);
        const uint32_t parity = static_cast<uint32_t>((i / STAGES) & 1);
        const bool ok = mbar_wait_bounded(&full[stage], parity, kWaitLimitNs);
        TileVec::In v[8];
        float amax = 0.0f;
        if (ok) {
            const uint8_t* tile = tiles + stage * kTileBytes;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint4 w = lds128(tile + (warp * 16 + 2 * k + row_in_load) * 256 + chunk * 16);
                v[k] = TileVec::In{{w.x, w.y, w.z, w.w}};
                amax = fmaxf(amax, TileVec::amax(v[k]));
            }
        }
        amax = warp_max<32>(amax);
        if (lane == 0) red[i & 1][warp] = amax;
        // One barrier per tile: every warp has its rows in registers (the stage
        // may be refilled) and its maximum in red[]; red[] alternates by tile
        // parity, so the next tile's writes cannot race these reads.
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(status, kStatusWaitTimeout);
            break;
        }
        if (tid == 0) {
            const int64_t t2 = t + STAGES * grid;
            if (t2 < ntiles) {
                issue(stage, t2);
                ++issued;
            }
        }
        float tile_amax = red[i & 1][0];
#pragma unroll
        for (int w = 1; w < kTmaThreads / 32; ++w) tile_amax = fmaxf(tile_amax, red[i & 1][w]);
        const float s = scale_from_amax<FMT>(tile_amax);
        const uint64_t s2 = f32x2(s, s);
        const int64_t tr = t / tiles_c;
        const int64_t tc = t - tr * tiles_c;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int64_t r = tr * 128 + warp * 16 + 2 * k + row_in_load;
            if (r < rows) st_stream(q + r * q_cols + tc * 16 + chunk, TileVec::cast<FMT>(v[k], s2));
        }
        if (tid == 0) scales[t] = s;
    }
    // On a timeout, wait (bounded) for the copies this CTA still has in flight
    // before its shared memory goes away.
    if (tid == 0) {
        for (int64_t j = i; j < issued; ++j) {
            const int stage = static_cast<int>(j % STAGES);
            mbar_wait_bounded(&full[stage], static_cast<uint32_t>((j / STAGES) & 1), kWaitLimitNs / 16);
        }
    }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult res;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &res) == cudaSuccess &&
            res == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

template <int FMT>
cudaError_t launch_tma_typed(const CUtensorMap& map, uint8_t* q, float* scales, int64_t rows, int64_t cols,
                             cudaStream_t st) {
    const int64_t ntiles = ((rows + 127) / 128) * (cols / 128);
    const size_t smem = static_cast<size_t>(kStages) * kTileBytes + kStages * sizeof(uint64_t) + 128;
    auto kern = k_quant_128x128_tma<FMT, kStages>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(ntiles, static_cast<int64_t>(device_sm_count()) * kCtasPerSm);
    unsigned int* status = device_status_word();
    if (status == nullptr) return cudaErrorInvalidValue;
    kern<<<static_cast<unsigned>(grid), kTmaThreads, smem, st>>>(map, reinterpret_cast<uint2*>(q), scales, rows,
                                                                 cols, ntiles, status);
    return cudaGetLastError();
}

}  // namespace

bool tma_128x128_supported(int dtype, int64_t rows, int64_t cols) {
    return dtype == 1 && cols % 128 == 0 && rows > 0 && rows < (int64_t(1) << 31) && cols < (int64_t(1) << 31) &&
           tensor_map_encoder() != nullptr;
}

cudaError_t launch_quant_128x128_tma(const void* x, int64_t rows, int64_t cols, int fmt, uint8_t* q, float* scales,
                                     cudaStream_t st) {
    auto encode = tensor_map_encoder();
    if (encode == nullptr) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};  // bytes between rows
    const cuuint32_t box[2] = {128, 128};
    const cuuint32_t elem_strides[2] = {1, 1};
    const CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(x), dims, strides, box,
                              elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    return fmt == kE4M3 ? launch_tma_typed<kE4M3>(map, q, scales, rows, cols, st)
                        : launch_tma_typed<kE5M2>(map, q, scales, rows, cols, st);
}

}  // namespace fp8q
