// quant_block_transpose.cu -- blockwise quantization with a transposed second
// output: q, scales = blockwise(x) and qt, scales_t = blockwise(x^T), from one
// read of x.
//
// Mixed-precision handbook, section "FP8 training", per_block: 1x128 blocks
// for activations, 128x128 blocks for weights, s = MAX / max(amax, eps) per
// block.  A weight-gradient (or data-gradient) GEMM reads its operand along
// the other dimension, so it needs the codes of x^T quantized with the same
// rule.  For 128x128 blocks x^T has the same blocks as x, transposed: qt is
// q^T and scales_t is scales^T.  For 1x128 blocks the blocks of x^T are the
// 128x1 columns of x, with scales of their own.
//
// One CTA per 128x128 tile (rows and cols multiples of 128).  The tile stays
// in registers, loaded as by the 128x128 block kernel (16 tile rows per warp,
// one lane vector per slice):
//   128x128  tile amax -> one scale; the codes go to q and into a shared code
//            tile, which is written out transposed into qt;
//   1x128    row amax over the lanes of a row (shuffles) -> q with the row
//            scales; column amax: per lane over its rows, then over the
//            warp's row groups (shuffles), then over the 8 warps (shared
//            memory) -> one scale per column, computed once by 128 threads;
//            the codes of x * column scale go into the shared tile and out
//            transposed into qt.
// Both casts are RN_fp32(x * s) then the saturating RNE cast, as everywhere.

#include <algorithm>
#include <atomic>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "launch_util.h"
#include "lane_vec.cuh"
#include "tensor_map.h"
#include "tile_transpose.cuh"
#include "umma.cuh"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Cast of one lane vector with a scale per element (column scales): cs[e] is
// the scale of element e, read from shared memory pair by pair.
// {cs[2p], cs[2p+1]} as packed fp32 operands (one 8-byte shared load).
[[maybe_unused]] __device__ __forceinline__ uint64_t pair(const float* cs, int p) {
    const float2 s = reinterpret_cast<const float2*>(cs)[p];
    return f32x2(s.x, s.y);
}

template <typename T, int BYTES>
struct PairCast;
template <int BYTES>
struct PairCast<uint16_t, BYTES> {
    using V = LaneVec<uint16_t, BYTES>;
    template <int FMT>
    static __device__ __forceinline__ typename V::Out cast(const typename V::In& v, const float* cs) {
        uint32_t c[V::kWords / 2];
#pragma unroll
        for (int k = 0; k < V::kWords / 2; ++k)
            c[k] = scale_cast_bf16x2<FMT>(v.w[2 * k], pair(cs, 2 * k)) |
                   (scale_cast_bf16x2<FMT>(v.w[2 * k + 1], pair(cs, 2 * k + 1)) << 16);
        return CodeWords<V::kWords / 2>::make(c);
    }
    // the same with the pairs already in registers: s2[p] = {cs[2p], cs[2p+1]}
    template <int FMT>
    static __device__ __forceinline__ typename V::Out cast_regs(const typename V::In& v,
                                                                const uint64_t (&s2)[V::kElems / 2]) {
        uint32_t c[V::kWords / 2];
#pragma unroll
        for (int k = 0; k < V::kWords / 2; ++k)
            c[k] = scale_cast_bf16x2<FMT>(v.w[2 * k], s2[2 * k]) |
                   (scale_cast_bf16x2<FMT>(v.w[2 * k + 1], s2[2 * k + 1]) << 16);
        return CodeWords<V::kWords / 2>::make(c);
    }
};
template <int BYTES>
struct PairCast<float, BYTES> {
    using V = LaneVec<float, BYTES>;
    template <int FMT>
    static __device__ __forceinline__ typename V::Out cast(const typename V::In& v, const float* cs) {
        uint32_t c[V::kWords / 4];
#pragma unroll
        for (int k = 0; k < V::kWords / 4; ++k)
            c[k] = scale_cast_f32x2<FMT>(v.w[4 * k], v.w[4 * k + 1], pair(cs, 2 * k)) |
                   (scale_cast_f32x2<FMT>(v.w[4 * k + 2], v.w[4 * k + 3], pair(cs, 2 * k + 1)) << 16);
        return CodeWords<V::kWords / 4>::make(c);
    }
    template <int FMT>
    static __device__ __forceinline__ typename V::Out cast_regs(const typename V::In& v,
                                                                const uint64_t (&s2)[V::kElems / 2]) {
        uint32_t c[V::kWords / 4];
#pragma unroll
        for (int k = 0; k < V::kWords / 4; ++k)
            c[k] = scale_cast_f32x2<FMT>(v.w[4 * k], v.w[4 * k + 1], s2[2 * k]) |
                   (scale_cast_f32x2<FMT>(v.w[4 * k + 2], v.w[4 * k + 3], s2[2 * k + 1]) << 16);
        return CodeWords<V::kWords / 4>::make(c);
    }
};

// |x| maxima of a lane's elements over its kLoads rows, then over the lanes
// that hold the same columns in the warp's other row groups; written (if
// `write`) to colmax[e] for element e of this lane's slice.  bf16 pairs reduce packed (exact); a NaN
// operand yields the other one, as in every amax of the library.
template <typename T, int BYTES>
struct ColMax;
template <int BYTES>
struct ColMax<uint16_t, BYTES> {
    using V = LaneVec<uint16_t, BYTES>;
    using G = TileGeom<uint16_t, BYTES>;
    static __device__ __forceinline__ void run(const typename V::In (&v)[G::kLoads], bool write, float* colmax) {
#pragma unroll
        for (int k = 0; k < V::kWords; ++k) {
            uint32_t m = v[0].w[k];
#pragma unroll
            for (int i = 1; i < G::kLoads; ++i) m = xabsmax_bf16x2(m, v[i].w[k]);
#pragma unroll
            for (int off = G::kVecPerRow; off < 32; off <<= 1)
                m = xabsmax_bf16x2(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
            m &= 0x7FFF7FFFu;
            if (write) {
                colmax[2 * k] = __uint_as_float(m << 16);
                colmax[2 * k + 1] = __uint_as_float(m & 0xFFFF0000u);
            }
        }
    }
    // The same maxima left packed, one word per column pair: colmax_w[k] holds columns 2k and 2k + 1 of
    // this lane's slice as two |bf16| halves, stored with 16-byte shared stores.
    static __device__ __forceinline__ void run_packed(const typename V::In (&v)[G::kLoads], bool write,
                                                      uint32_t* colmax_w) {
        uint32_t mw[V::kWords];
#pragma unroll
        for (int k = 0; k < V::kWords; ++k) {
            uint32_t m = v[0].w[k];
#pragma unroll
            for (int i = 1; i < G::kLoads; ++i) m = xabsmax_bf16x2(m, v[i].w[k]);
#pragma unroll
            for (int off = G::kVecPerRow; off < 32; off <<= 1)
                m = xabsmax_bf16x2(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
            mw[k] = m & 0x7FFF7FFFu;
        }
        if (write) {
#pragma unroll
            for (int k4 = 0; k4 < V::kWords / 4; ++k4)
                reinterpret_cast<uint4*>(colmax_w)[k4] = make_uint4(mw[4 * k4], mw[4 * k4 + 1], mw[4 * k4 + 2],
                                                                    mw[4 * k4 + 3]);
        }
    }
};
template <int BYTES>
struct ColMax<float, BYTES> {
    using V = LaneVec<float, BYTES>;
    using G = TileGeom<float, BYTES>;
    static __device__ __forceinline__ void run(const typename V::In (&v)[G::kLoads], bool write, float* colmax) {
#pragma unroll
        for (int k = 0; k < V::kWords; ++k) {
            float m = fabsf(__uint_as_float(v[0].w[k]));
#pragma unroll
            for (int i = 1; i < G::kLoads; ++i) m = fmaxf(m, fabsf(__uint_as_float(v[i].w[k])));
#pragma unroll
            for (int off = G::kVecPerRow; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
            if (write) colmax[k] = m;
        }
    }
};

// MODE 0: 1x128 blocks (row scales for q, column scales for qt);
// MODE 1: 128x128 blocks (one scale per tile for both).
// 1x128 reads its tile a second time, from L2, for the column cast instead
// of holding it in registers through the row pass and the column pass; with
// that (and the row scales' divisions shared among a row's lanes) the kernel
// fits the register cap of 4 CTAs per SM without spilling (bf16; an fp32
// tile is twice the registers and keeps the cap of 2).  Measured on B200,
// bf16 activations 16384x7168, 1x128: 4954 GB/s holding the tile with a cap
// of 2 CTAs (4544 with a cap of 3); with the second read issued after the
// column pass's barriers 4598 / 5162 / 5210 GB/s for caps of 2 / 3 / 4 CTAs,
// and 5437 GB/s with it issued before them (RELOAD 2), so that the loads are
// in flight across the barriers.  The column cast takes this lane's 16
// column scales into registers once (SCALE_REGS).  Keeping bf16 column
// maxima as packed |bf16| pairs through shared memory (PACKED_PART: two
// 16-byte stores per writing lane instead of 16 scalar ones, no unpacking)
// gives 5567-5573 GB/s against 5429-5431.  Every warp forming the column
// scales its lanes need (SCALES_IN_WARP: 4 per lane, shared by shuffles)
// instead of 128 threads forming them behind a second barrier: 5658-5663
// against 5590-5594 GB/s.  128x128: 6462 GB/s (98.7 % of the copy peak)
// with 3 or 4 CTAs.
#ifndef FP8Q_BT_TMA
#define FP8Q_BT_TMA 0
#endif
#ifndef FP8Q_BLOCK_TRANSPOSE_RELOAD
#define FP8Q_BLOCK_TRANSPOSE_RELOAD 2
#endif
#ifndef FP8Q_BLOCK_TRANSPOSE_SCALE_REGS
#define FP8Q_BLOCK_TRANSPOSE_SCALE_REGS 1
#endif
// bf16 column maxima kept as packed |bf16| pairs through shared memory
#ifndef FP8Q_BLOCK_TRANSPOSE_PACKED_PART
#define FP8Q_BLOCK_TRANSPOSE_PACKED_PART 1
#endif
// 1x128, bf16 with 32-byte lanes: each warp forms the column scales it needs (no second barrier).
#ifndef FP8Q_BT_SCALES_IN_WARP
#define FP8Q_BT_SCALES_IN_WARP 1
#endif
#ifndef FP8Q_BLOCK_TRANSPOSE_1X128_MIN_CTAS
#define FP8Q_BLOCK_TRANSPOSE_1X128_MIN_CTAS 4
#endif
#ifndef FP8Q_BLOCK_TRANSPOSE_128X128_MIN_CTAS
#define FP8Q_BLOCK_TRANSPOSE_128X128_MIN_CTAS 3
#endif

template <typename T, int FMT, int BYTES, int MODE>
__global__ void __launch_bounds__(kThreads, MODE == 1               ? FP8Q_BLOCK_TRANSPOSE_128X128_MIN_CTAS
                                           : sizeof(T) == 2         ? FP8Q_BLOCK_TRANSPOSE_1X128_MIN_CTAS
                                                                    : 2)
k_quant_block_transpose(const T* __restrict__ x, int64_t rows, int64_t cols, uint8_t* __restrict__ q,
                        float* __restrict__ scales, uint8_t* __restrict__ qt, float* __restrict__ scales_t) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    using G = TileGeom<T, BYTES>;
    __shared__ __align__(16) uint8_t tile[kTT * kTT];
    __shared__ __align__(16) float part[kWarps][kTT];  // per-warp column maxima (MODE 0); warp maxima (MODE 1)
    // bf16, MODE 0 with packed partials: the same storage as [kWarps][kTT / 2] words of |bf16| pairs
    uint32_t (*part_w)[kTT] = reinterpret_cast<uint32_t (*)[kTT]>(part);
    constexpr bool kPackedPart = FP8Q_BLOCK_TRANSPOSE_PACKED_PART && sizeof(T) == 2;
    __shared__ __align__(16) float col_scale[kTT];

    const int64_t tiles_c = cols / kTT, tiles_r = rows / kTT;
    const int64_t tr = blockIdx.x / tiles_c;
    const int64_t tc = blockIdx.x - tr * tiles_c;
    const int64_t r0 = tr * kTT, c0 = tc * kTT;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lr0 = warp * 16 + lane / G::kVecPerRow, vec_in_row = lane % G::kVecPerRow;
    const auto* xv = reinterpret_cast<const typename V::In*>(x + (r0 + lr0) * cols + c0) + vec_in_row;
    const int64_t vstride = cols / V::kElems * G::kRowsPerLoad;  // lane vectors between this lane's rows
    typename V::In v[G::kLoads];
#pragma unroll
    for (int i = 0; i < G::kLoads; ++i) v[i] = ld_words_stream(xv + i * vstride);

    if (MODE == 1) {
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i) a = fmaxf(a, V::amax(v[i]));
        a = warp_max<32>(a);
        if (lane == 0) part[0][warp] = a;
        __syncthreads();
        float ta = part[0][0];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) ta = fmaxf(ta, part[0][w]);
        const float s = scale_from_amax<FMT>(ta);
        float unused = 0.0f;
        tile_cast<T, FMT, BYTES, false>(v, f32x2(s, s), q, cols, r0, c0, tile, lr0, vec_in_row, unused);
        if (threadIdx.x == 0) {
            scales[tr * tiles_c + tc] = s;
            scales_t[tc * tiles_r + tr] = s;
        }
    } else {
        // q: one scale per tile row.  The row's kVecPerRow lanes reduce its
        // amax together; lane j of the row computes the scale of load j (one
        // division per lane) and the row's lanes fetch the rest by shuffles.
        float ra[G::kLoads];
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i) ra[i] = warp_max<G::kVecPerRow>(V::amax(v[i]));
        float mine = 0.0f;
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i)
            if (i % G::kVecPerRow == vec_in_row) mine = ra[i];
        const float s_mine = scale_from_amax<FMT>(mine);
        const int group = lane - vec_in_row;  // first lane of this row
#if FP8Q_BLOCK_TRANSPOSE_RELOAD == 3
        // qt's column maxima first; then each row is cast to q and its registers
        // reloaded from L2 at once, so the reloads start as early as they can
        ColMax<T, BYTES>::run(v, lane < G::kVecPerRow, &part[warp][vec_in_row * V::kElems]);
#endif
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i) {
            const float s = __shfl_sync(0xFFFFFFFFu, s_mine, group + i % G::kVecPerRow);
            const int lr = lr0 + i * G::kRowsPerLoad;
            st_stream(reinterpret_cast<typename V::Out*>(q + (r0 + lr) * cols + c0) + vec_in_row,
                      V::template cast<FMT>(v[i], f32x2(s, s)));
            if (vec_in_row == 0) scales[(r0 + lr) * tiles_c + tc] = s;
#if FP8Q_BLOCK_TRANSPOSE_RELOAD == 3
            v[i] = ld_words_stream(xv + i * vstride);
#endif
        }
#if FP8Q_BLOCK_TRANSPOSE_RELOAD != 3
        // qt: one scale per tile column
        if constexpr (kPackedPart)
            ColMax<T, BYTES>::run_packed(v, lane < G::kVecPerRow, &part_w[warp][vec_in_row * V::kElems / 2]);
        else
            ColMax<T, BYTES>::run(v, lane < G::kVecPerRow, &part[warp][vec_in_row * V::kElems]);
#endif
#if FP8Q_BLOCK_TRANSPOSE_RELOAD == 2
        // the tile again, from L2, issued now so that the loads are in flight
        // across the two barriers of the column pass
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i) v[i] = ld_words_stream(xv + i * vstride);
#endif
#if FP8Q_BT_SCALES_IN_WARP
        if constexpr (kPackedPart && BYTES == 32 && FP8Q_BLOCK_TRANSPOSE_SCALE_REGS) {
            __syncthreads();
            // Every warp forms the column scales its lanes need, with no second barrier: the 4 lanes
            // that hold the same 16 columns (one per row group) each reduce 4 of them over the 8 warps'
            // packed maxima and share them by shuffles.  Warp 0 stores scales_t.
            const int rowgrp = lane / G::kVecPerRow;
            const int w0 = vec_in_row * (V::kElems / 2) + rowgrp * 2;
            uint32_t ma = part_w[0][w0], mb = part_w[0][w0 + 1];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) {
                ma = xabsmax_bf16x2(ma, part_w[w][w0]);
                mb = xabsmax_bf16x2(mb, part_w[w][w0 + 1]);
            }
            float s4[4] = {scale_from_amax<FMT>(__uint_as_float(ma << 16)),
                           scale_from_amax<FMT>(__uint_as_float(ma & 0xFFFF0000u)),
                           scale_from_amax<FMT>(__uint_as_float(mb << 16)),
                           scale_from_amax<FMT>(__uint_as_float(mb & 0xFFFF0000u))};
            if (warp == 0) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    scales_t[(c0 + vec_in_row * V::kElems + rowgrp * 4 + k) * tiles_r + tr] = s4[k];
            }
            uint64_t cs2[V::kElems / 2];
#pragma unroll
            for (int g = 0; g < V::kElems / 4; ++g) {
                const int src = g * G::kVecPerRow + vec_in_row;
                const float a = __shfl_sync(0xFFFFFFFFu, s4[0], src), b = __shfl_sync(0xFFFFFFFFu, s4[1], src);
                const float c_ = __shfl_sync(0xFFFFFFFFu, s4[2], src), d = __shfl_sync(0xFFFFFFFFu, s4[3], src);
                cs2[2 * g] = f32x2(a, b);
                cs2[2 * g + 1] = f32x2(c_, d);
            }
#pragma unroll
            for (int i = 0; i < G::kLoads; ++i) {
                const int lr = lr0 + i * G::kRowsPerLoad;
                *reinterpret_cast<typename V::Out*>(tile + tile_off(lr, vec_in_row * V::kElems)) =
                    PairCast<T, BYTES>::template cast_regs<FMT>(v[i], cs2);
            }
        } else
#endif
        {
        __syncthreads();
        if (threadIdx.x < kTT) {
            const int c = threadIdx.x;
            float m;
            if constexpr (kPackedPart) {
                uint32_t mw = part_w[0][c >> 1];
#pragma unroll
                for (int w = 1; w < kWarps; ++w) mw = xabsmax_bf16x2(mw, part_w[w][c >> 1]);
                m = __uint_as_float((c & 1) ? (mw & 0xFFFF0000u) : (mw << 16));
            } else {
                m = part[0][c];
#pragma unroll
                for (int w = 1; w < kWarps; ++w) m = fmaxf(m, part[w][c]);
            }
            const float s = scale_from_amax<FMT>(m);
            col_scale[c] = s;
            scales_t[(c0 + c) * tiles_r + tr] = s;
        }
        __syncthreads();
        const float* cs = col_scale + vec_in_row * V::kElems;
#if FP8Q_BLOCK_TRANSPOSE_RELOAD == 1
        // the tile again, from L2 (it was read a moment ago), instead of
        // holding it in registers across the two barriers above
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i) v[i] = ld_words_stream(xv + i * vstride);
#endif
#if FP8Q_BLOCK_TRANSPOSE_SCALE_REGS
        // this lane's column scales are the same for all its rows: into registers once, as packed pairs
        uint64_t cs2[V::kElems / 2];
#pragma unroll
        for (int p4 = 0; p4 < V::kElems / 4; ++p4) {
            const float4 c4 = reinterpret_cast<const float4*>(cs)[p4];
            cs2[2 * p4] = f32x2(c4.x, c4.y);
            cs2[2 * p4 + 1] = f32x2(c4.z, c4.w);
        }
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i) {
            const int lr = lr0 + i * G::kRowsPerLoad;
            *reinterpret_cast<typename V::Out*>(tile + tile_off(lr, vec_in_row * V::kElems)) =
                PairCast<T, BYTES>::template cast_regs<FMT>(v[i], cs2);
        }
#else
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i) {
            const int lr = lr0 + i * G::kRowsPerLoad;
            *reinterpret_cast<typename V::Out*>(tile + tile_off(lr, vec_in_row * V::kElems)) =
                PairCast<T, BYTES>::template cast<FMT>(v[i], cs);
        }
#endif
        }
    }
    __syncthreads();
    tile_transpose_out(tile, qt, rows, r0, c0, lane, warp);
}

#if FP8Q_BT_TMA
// ---------------------------------------------------------------------------
// 1x128 blocks of bf16 x and x^T, TMA-staged and persistent: the measured
// alternative to the register-tile kernel above, compiled in only with
// -DFP8Q_BT_TMA=1.
//
// The register-tile kernel spends most of a tile's time computing (two
// casts, the row and column reductions, three barriers) with nothing in
// flight to HBM, and its column pass reads the tile a second time from L2.
// Here each CTA walks tiles first, first + step, ... and keeps the next
// kStages tiles in flight: a 2-D TMA load (no multicast) brings each 128x128
// bf16 tile (32 KiB) into a shared-memory stage, completing on the stage's
// mbarrier, and is issued for tile i + kStages as soon as tile i's last read
// of the stage is behind a barrier.  Both passes read the tile from shared
// memory, with the lane geometry of the register kernel (16 tile rows per
// warp, one 32-byte slice per lane and load), so the arithmetic is the same:
// row amax -> row scale -> q; column amax (lane, warp row groups, warps) ->
// column scale -> codes into the swizzled code tile -> qt.
// Measured on B200 (bf16 activations 16384x7168): 3674 GB/s with 2 stages
// and 2 CTAs per SM, 3263 GB/s with 3 stages and 1 CTA, against 5204 GB/s
// for the register kernel.  The stages and 118 registers per thread leave 16
// warps per SM, a quarter of the slots, for a kernel whose per-tile work is
// long chains of dependent instructions: issue activity falls from 48 % to
// 32 % of peak and DRAM throughput from 54 % to 39 % (ncu, cold L2).
// Waits are bounded; a wait that runs out sets the device status bit, the
// CTA stops, and it waits (bounded) for its loads in flight before it exits.
// ---------------------------------------------------------------------------
#ifndef FP8Q_BT_TMA_STAGES
#define FP8Q_BT_TMA_STAGES 2
#endif
#ifndef FP8Q_BT_TMA_CTAS
#define FP8Q_BT_TMA_CTAS 2
#endif
constexpr int kBtStages = FP8Q_BT_TMA_STAGES;
constexpr int kBtTileBytes = kTT * kTT * 2;  // one bf16 tile
struct BtSmem {
    static constexpr int kStage = 0;
    static constexpr int kCode = kBtStages * kBtTileBytes;
    static constexpr int kPart = kCode + kTT * kTT;
    static constexpr int kColScale = kPart + kWarps * kTT * 4;
    static constexpr int kBars = kColScale + kTT * 4;
    static constexpr int kBytes = kBars + kBtStages * 8;
    static constexpr int kAlloc = kBytes + 128;  // alignment slack
};

__device__ __forceinline__ Words<8> lds32(const uint8_t* p) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint4 b = *reinterpret_cast<const uint4*>(p + 16);
    return Words<8>{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, FP8Q_BT_TMA_CTAS)
k_quant_block_transpose_tma(const __grid_constant__ CUtensorMap map_x, int64_t rows, int64_t cols,
                            uint8_t* __restrict__ q, float* __restrict__ scales, uint8_t* __restrict__ qt,
                            float* __restrict__ scales_t, unsigned int* status) {
    using V = LaneVec<uint16_t, 32>;
    using G = TileGeom<uint16_t, 32>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t* tile = sm + BtSmem::kCode;
    float (*part)[kTT] = reinterpret_cast<float (*)[kTT]>(sm + BtSmem::kPart);
    float* col_scale = reinterpret_cast<float*>(sm + BtSmem::kColScale);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + BtSmem::kBars);

    const int64_t tiles_c = cols / kTT, tiles_r = rows / kTT;
    const int64_t tiles = tiles_r * tiles_c;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lr0 = warp * 16 + lane / G::kVecPerRow, vec_in_row = lane % G::kVecPerRow;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBtStages; ++s) umma::mbar_init(&full[s], 1);
        umma::fence_mbar_init();
    }
    __syncthreads();
    pdl_enter();  // x may come from the previous kernel

    auto issue = [&](int64_t t, int s) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        umma::mbar_arrive_expect_tx(&full[s], kBtTileBytes);
        umma::tma_load_2d(sm + BtSmem::kStage + s * kBtTileBytes, &map_x, &full[s], static_cast<int>(tc * kTT),
                          static_cast<int>(tr * kTT));
    };
    if (threadIdx.x == 0) {
        for (int s = 0; s < kBtStages; ++s) {
            const int64_t t = blockIdx.x + static_cast<int64_t>(s) * gridDim.x;
            if (t < tiles) issue(t, s);
        }
    }

    bool timed_out = false;
    int i = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int s = i % kBtStages;
        const uint32_t parity = static_cast<uint32_t>(i / kBtStages) & 1u;
        const bool ok = umma::mbar_wait(&full[s], parity, kWaitLimitNs);
        const uint8_t* stage = sm + BtSmem::kStage + s * kBtTileBytes;
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        const int64_t r0 = tr * kTT, c0 = tc * kTT;

        typename V::In v[G::kLoads];
        if (ok) {
#pragma unroll
            for (int k = 0; k < G::kLoads; ++k)
                v[k] = lds32(stage + (lr0 + k * G::kRowsPerLoad) * (kTT * 2) + vec_in_row * 32);
            // q: one scale per tile row, as in the register kernel
            float ra[G::kLoads];
#pragma unroll
            for (int k = 0; k < G::kLoads; ++k) ra[k] = warp_max<G::kVecPerRow>(V::amax(v[k]));
            float mine = 0.0f;
#pragma unroll
            for (int k = 0; k < G::kLoads; ++k)
                if (k % G::kVecPerRow == vec_in_row) mine = ra[k];
            const float s_mine = scale_from_amax<FMT>(mine);
            const int group = lane - vec_in_row;
#pragma unroll
            for (int k = 0; k < G::kLoads; ++k) {
                const float sc = __shfl_sync(0xFFFFFFFFu, s_mine, group + k % G::kVecPerRow);
                const int lr = lr0 + k * G::kRowsPerLoad;
                st_stream(reinterpret_cast<typename V::Out*>(q + (r0 + lr) * cols + c0) + vec_in_row,
                          V::template cast<FMT>(v[k], f32x2(sc, sc)));
                if (vec_in_row == 0) scales[(r0 + lr) * tiles_c + tc] = sc;
            }
            ColMax<uint16_t, 32>::run(v, lane < G::kVecPerRow, &part[warp][vec_in_row * V::kElems]);
        }
        if (__syncthreads_or(!ok)) {
            timed_out = true;
            break;
        }
        if (threadIdx.x < kTT) {
            const int c = threadIdx.x;
            float m = part[0][c];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) m = fmaxf(m, part[w][c]);
            const float sc = scale_from_amax<FMT>(m);
            col_scale[c] = sc;
            scales_t[(c0 + c) * tiles_r + tr] = sc;
        }
        __syncthreads();
        const float* cs = col_scale + vec_in_row * V::kElems;
#pragma unroll
        for (int k = 0; k < G::kLoads; ++k) {
            const int lr = lr0 + k * G::kRowsPerLoad;
            const typename V::In w = lds32(stage + lr * (kTT * 2) + vec_in_row * 32);
            *reinterpret_cast<typename V::Out*>(tile + tile_off(lr, vec_in_row * V::kElems)) =
                PairCast<uint16_t, 32>::template cast<FMT>(w, cs);
        }
        __syncthreads();  // the stage is read and the code tile complete
        if (threadIdx.x == 0) {
            const int64_t tn = t + static_cast<int64_t>(kBtStages) * gridDim.x;
            if (tn < tiles) issue(tn, s);
        }
        tile_transpose_out(tile, qt, rows, r0, c0, lane, warp);
    }
    if (timed_out) {
        if (threadIdx.x == 0) {
            atomicOr(status, kStatusWaitTimeout);
            // loads may still be landing in this CTA's shared memory: let them finish (bounded)
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 1000000ull) {
            }
        }
        __syncthreads();
    }
}

template <int FMT>
cudaError_t launch_bt_tma(const void* x, int64_t rows, int64_t cols, uint8_t* q, float* scales, uint8_t* qt,
                          float* scales_t, cudaStream_t st, bool* launched) {
    *launched = false;
    const int64_t tiles = (rows / kTT) * (cols / kTT);
    if (rows > 0x7FFFFFFF || cols > 0x7FFFFFFF) return cudaSuccess;  // TMA coordinates are 32-bit
    CUtensorMap map;
    if (!make_bf16_tile_map(&map, x, rows, cols, kTT, kTT)) return cudaSuccess;
    unsigned int* status = device_status_word();
    if (status == nullptr) return cudaSuccess;
    auto kern = k_quant_block_transpose_tma<FMT>;
    // The shared-memory opt-in and the co-resident grid, once per device.
    static std::atomic<int> resident[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
    int units = resident[dev].load(std::memory_order_acquire);
    if (units <= 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BtSmem::kAlloc);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, BtSmem::kAlloc);
        if (e != cudaSuccess) return e;
        units = std::max(1, per_sm) * device_sm_count();
        resident[dev].store(units, std::memory_order_release);
    }
    const int64_t grid = std::min<int64_t>(tiles, units);
    const cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), BtSmem::kAlloc, st,
                                        map, rows, cols, q, scales, qt, scales_t, status);
    if (e == cudaSuccess) *launched = true;
    return e;
}
#endif  // FP8Q_BT_TMA

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <typename T, int FMT, int BYTES>
cudaError_t launch_typed(const void* x, int64_t rows, int64_t cols, int block_rows, uint8_t* q, float* scales,
                         uint8_t* qt, float* scales_t, cudaStream_t st) {
    const int64_t tiles = (rows / kTT) * (cols / kTT);
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(tiles));
    const cudaError_t e =
        block_rows == 1
            ? launch_kernel(k_quant_block_transpose<T, FMT, BYTES, 0>, grid, dim3(kThreads), 0, st,
                            static_cast<const T*>(x), rows, cols, q, scales, qt, scales_t)
            : launch_kernel(k_quant_block_transpose<T, FMT, BYTES, 1>, grid, dim3(kThreads), 0, st,
                            static_cast<const T*>(x), rows, cols, q, scales, qt, scales_t);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t launch_width(const void* x, int64_t rows, int64_t cols, int block_rows, uint8_t* q, float* scales,
                         uint8_t* qt, float* scales_t, cudaStream_t st) {
    // 256-bit lanes when every tile row starts on a 32-byte boundary
    if (aligned32(x) && (cols * static_cast<int64_t>(sizeof(T))) % 32 == 0)
        return launch_typed<T, FMT, 32>(x, rows, cols, block_rows, q, scales, qt, scales_t, st);
    return launch_typed<T, FMT, 16>(x, rows, cols, block_rows, q, scales, qt, scales_t, st);
}

}  // namespace

cudaError_t launch_quant_block_transpose(const void* x, int dtype, int64_t rows, int64_t cols, int block_rows,
                                         int fmt, uint8_t* q, float* scales, uint8_t* qt, float* scales_t,
                                         cudaStream_t st) {
    if (rows == 0 || cols == 0) return cudaSuccess;
#if FP8Q_BT_TMA
    if (dtype == 1 && block_rows == 1) {
        // bf16 in 1x128 blocks: the TMA-staged persistent kernel, where the driver offers tensor maps
        bool launched = false;
        const cudaError_t e = fmt == kE4M3 ? launch_bt_tma<kE4M3>(x, rows, cols, q, scales, qt, scales_t, st, &launched)
                                           : launch_bt_tma<kE5M2>(x, rows, cols, q, scales, qt, scales_t, st, &launched);
        if (e != cudaSuccess || launched) return e;
    }
#endif
    if (dtype == 1)
        return fmt == kE4M3 ? launch_width<uint16_t, kE4M3>(x, rows, cols, block_rows, q, scales, qt, scales_t, st)
                            : launch_width<uint16_t, kE5M2>(x, rows, cols, block_rows, q, scales, qt, scales_t, st);
    return fmt == kE4M3 ? launch_width<float, kE4M3>(x, rows, cols, block_rows, q, scales, qt, scales_t, st)
                        : launch_width<float, kE5M2>(x, rows, cols, block_rows, q, scales, qt, scales_t, st);
}

}  // namespace fp8q
