// quant_tensor.cu -- per-tensor FP8 quantization kernels.
//
// Mixed-precision handbook, section "FP8 training", per_tensor: one scale for
// the whole tensor.  PyTorch-FP8 page s4.1 (scale = max_val / amax) and s4.2
// (delayed scaling: the scale comes from earlier steps' amax, so the cast
// needs no global reduction first).
//
// Current scaling is two grid-wide passes after k_zero_f32 clears the
// caller's amax_out: k_tensor_amax (at most one atomicMax per CTA into
// amax_out), then k_tensor_cast, which turns that amax into s in every CTA.  The cast pass takes its chunks in the
// reverse order of the amax pass, so its first reads find the most recently
// read data still in L2.  Delayed scaling is one pass: cast with the given s
// and reduce this step's amax from the same registers.  Each CTA owns one
// contiguous chunk and issues all its loads before computing.

#include <algorithm>
#include <atomic>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "history_update.cuh"
#include "launch_util.h"
#include "lane_vec.cuh"
#include "tile_transpose.cuh"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
// Lane vectors loaded per trip per thread.
#ifndef FP8Q_TENSOR_UNROLL
#define FP8Q_TENSOR_UNROLL 4
#endif
constexpr int kUnroll = FP8Q_TENSOR_UNROLL;

template <typename T>
__device__ __forceinline__ float load_scalar(const T* p, int i);
template <>
__device__ __forceinline__ float load_scalar<uint16_t>(const uint16_t* p, int i) {
    return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
}
template <>
__device__ __forceinline__ float load_scalar<float>(const float* p, int i) { return p[i]; }

// CTA-wide max, then at most one atomicMax per CTA: the atomic is skipped when
// the running maximum already read back is at least as large (a stale read can
// only cost an extra atomic, never lose the maximum).
__device__ __forceinline__ void cta_amax_to_global(float a, float* amax_out) {
    __shared__ float warp_amax[kThreads / 32];
    a = warp_max<32>(a);
    if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = warp_amax[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, warp_amax[w]);
        float seen;
        asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(seen) : "l"(amax_out) : "memory");
        if (!(m <= seen)) atomic_max_nonneg(amax_out, m);
    }
}

// Pass 1 of current scaling.  Each CTA reduces kThreads x kUnroll consecutive
// lane vectors; x's tail_n trailing elements (< one vector) go to CTA 0.
template <typename T, int BYTES>
__global__ void __launch_bounds__(kThreads)
k_tensor_amax(const typename LaneVec<T, BYTES>::In* __restrict__ x, int64_t nvec, const T* __restrict__ tail,
              int tail_n, float* __restrict__ amax_out) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads * kUnroll + threadIdx.x;
    typename V::In v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        v[u] = (i < nvec) ? ld_words_stream(x + i) : V::zero();
    }
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) a = fmaxf(a, V::amax(v[u]));
    if (blockIdx.x == 0 && threadIdx.x < tail_n) a = fmaxf(a, fabsf(load_scalar(tail, threadIdx.x)));
    cta_amax_to_global(a, amax_out);
}

// Pass 2 of current scaling (DELAYED = false: s from *amax_in), or the single
// pass of delayed scaling (DELAYED = true: s = *scale_in; WITH_AMAX also
// reduces amax(x) into *amax_out).  CTAs take their chunks last-to-first.
template <typename T, int FMT, int BYTES, bool DELAYED, bool WITH_AMAX>
__global__ void __launch_bounds__(kThreads)
k_tensor_cast(const typename LaneVec<T, BYTES>::In* __restrict__ x, int64_t nvec, const T* __restrict__ tail,
              int tail_n, const float* scale_in, const float* __restrict__ amax_in,
              typename LaneVec<T, BYTES>::Out* __restrict__ q, uint8_t* __restrict__ q_tail, float* scale_out,
              float* __restrict__ amax_out) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    const int64_t chunk = static_cast<int64_t>(gridDim.x) - 1 - blockIdx.x;
    const int64_t base = chunk * kThreads * kUnroll + threadIdx.x;
    typename V::In v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        v[u] = (i < nvec) ? ld_words_stream(x + i) : V::zero();
    }
    const float s = DELAYED ? *scale_in : scale_from_amax<FMT>(*amax_in);
    const uint64_t s2 = f32x2(s, s);
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        if (WITH_AMAX) a = fmaxf(a, V::amax(v[u]));
        if (i < nvec) st_stream(q + i, V::template cast<FMT>(v[u], s2));
    }
    if (blockIdx.x == 0 && threadIdx.x < tail_n) {
        const float xv = load_scalar(tail, threadIdx.x);
        if (WITH_AMAX) a = fmaxf(a, fabsf(xv));
        q_tail[threadIdx.x] = static_cast<uint8_t>(cvt_fp8x2<FMT>(__fmul_rn(xv, s), 0.0f) & 0xFFu);
    }
    if (WITH_AMAX) cta_amax_to_global(a, amax_out);
    // Written after every read of *scale_in in this CTA (the caller may pass
    // the same pointer for both; other CTAs read the same value either way).
    if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = s;
}

// ---------------------------------------------------------------------------
// One step of delayed scaling in one launch: the cast with the given scale,
// amax(x) from the same registers, and -- in whichever CTA finishes last --
// the amax-history update that produces the next step's scale.  The same
// result as the delayed cast followed by the history update kernel.
//
// Every CTA folds its amax into ws->amax_bits, then counts itself in
// ws->arrivals (fence first); the CTA that takes the count to gridDim.x is
// last, so it sees every CTA's amax.  It writes amax_out and scale_used, runs
// the history update (one warp), and puts the workspace back to zero.  No CTA
// waits for another.  *scale is read by every CTA before it counts itself and
// written only by the last one, so it is updated in place.
// ---------------------------------------------------------------------------
struct StepWorkspace {
    unsigned int arrivals;
    unsigned int amax_bits;
    unsigned int unused[2];
};
static_assert(sizeof(StepWorkspace) == 16, "workspace layout");

// One CTA's chunk `chunk` of `nchunks` (the body of k_tensor_cast_delayed_step,
// also run by the grouped kernel for each tensor's chunks).
template <typename T, int FMT, int BYTES>
__device__ __forceinline__ void delayed_step_cta(const typename LaneVec<T, BYTES>::In* __restrict__ x, int64_t nvec,
                                                 const T* __restrict__ tail, int tail_n, float* scale,
                                                 typename LaneVec<T, BYTES>::Out* __restrict__ q,
                                                 uint8_t* __restrict__ q_tail, float* __restrict__ scale_used,
                                                 float* __restrict__ amax_out, float* history, int32_t* state,
                                                 int window, int algo, float alpha, float margin, StepWorkspace* ws,
                                                 int64_t chunk, int64_t nchunks) {
    using V = LaneVec<T, BYTES>;
    __shared__ float warp_amax[kThreads / 32];
    const int64_t base = chunk * kThreads * kUnroll + threadIdx.x;
    typename V::In v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        v[u] = (i < nvec) ? ld_words_stream(x + i) : V::zero();
    }
    const float s = *scale;
    const uint64_t s2 = f32x2(s, s);
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        a = fmaxf(a, V::amax(v[u]));
        if (i < nvec) st_stream(q + i, V::template cast<FMT>(v[u], s2));
    }
    if (chunk == 0 && threadIdx.x < tail_n) {
        const float xv = load_scalar(tail, threadIdx.x);
        a = fmaxf(a, fabsf(xv));
        q_tail[threadIdx.x] = static_cast<uint8_t>(cvt_fp8x2<FMT>(__fmul_rn(xv, s), 0.0f) & 0xFFu);
    }
    a = warp_max<32>(a);
    if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = a;
    __syncthreads();
    // Only warp 0 goes on: the other warps' slots free up for the next CTAs.
    if (threadIdx.x >= 32) return;
    int is_last = 0;
    if (threadIdx.x == 0) {
        float m = warp_amax[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, warp_amax[w]);
        atomicMax(&ws->amax_bits, __float_as_uint(m));  // non-negative floats order as their bits
        __threadfence();
        is_last = (atomicAdd(&ws->arrivals, 1u) == static_cast<unsigned int>(nchunks - 1));
    }
    if (!__shfl_sync(0xFFFFFFFFu, is_last, 0)) return;
    __threadfence();
    const float amax = __uint_as_float(atomicAdd(&ws->amax_bits, 0u));
    if (threadIdx.x == 0) {
        *amax_out = amax;
        *scale_used = s;
    }
    history_update_warp<FMT>(history, state, window, amax, scale, algo, alpha, margin);
    if (threadIdx.x == 0) {
        ws->amax_bits = 0u;
        ws->arrivals = 0u;
    }
}

template <typename T, int FMT, int BYTES>
__global__ void __launch_bounds__(kThreads)
k_tensor_cast_delayed_step(const typename LaneVec<T, BYTES>::In* __restrict__ x, int64_t nvec,
                           const T* __restrict__ tail, int tail_n, float* scale,
                           typename LaneVec<T, BYTES>::Out* __restrict__ q, uint8_t* __restrict__ q_tail,
                           float* __restrict__ scale_used, float* __restrict__ amax_out, float* history,
                           int32_t* state, int window, int algo, float alpha, float margin, StepWorkspace* ws) {
    pdl_enter();
    delayed_step_cta<T, FMT, BYTES>(x, nvec, tail, tail_n, scale, q, q_tail, scale_used, amax_out, history, state,
                                    window, algo, alpha, margin, ws, blockIdx.x, gridDim.x);
}

// Many tensors' delayed steps in one launch: each tensor's chunks are numbered
// consecutively across the group, a CTA finds its tensor by binary search
// over the start indices (kernel parameters), and each tensor has its own
// 16-byte workspace slot, so its last CTA updates its history.
constexpr int kStepGroupMax = 128;  // tensors per launch (a 9.3 KiB parameter block; the limit is 32 KiB)

struct StepTable {
    int count;
    int window, algo;
    float alpha, margin;
    StepWorkspace* ws;              // slot of this launch's first tensor
    int64_t start[kStepGroupMax + 1];
    DelayedTensor e[kStepGroupMax];
};
static_assert(sizeof(StepTable) <= 16384, "the grouped step's parameter block must stay well inside 32 KiB");

template <typename T, int FMT, int BYTES>
__global__ void __launch_bounds__(kThreads)
k_tensor_cast_delayed_step_grouped(const __grid_constant__ StepTable tab) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    const int64_t b = blockIdx.x;
    int lo = 0, hi = tab.count;  // start[lo] <= b < start[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tab.start[mid] <= b) lo = mid;
        else hi = mid;
    }
    const DelayedTensor& e = tab.e[lo];
    const int64_t nvec = e.n / V::kElems;
    const int tail_n = static_cast<int>(e.n - nvec * V::kElems);
    delayed_step_cta<T, FMT, BYTES>(static_cast<const typename V::In*>(e.x), nvec,
                                    static_cast<const T*>(e.x) + nvec * V::kElems, tail_n, e.scale,
                                    reinterpret_cast<typename V::Out*>(e.q), e.q + nvec * V::kElems, e.scale_used,
                                    e.amax_out, e.history, e.state, tab.window, tab.algo, tab.alpha, tab.margin,
                                    tab.ws + lo, b - tab.start[lo], tab.start[lo + 1] - tab.start[lo]);
}

// Per-tensor current scaling of many tensors in three launches: every
// tensor's amax_out is cleared, then one amax pass and one cast pass run over
// all tensors' chunks, numbered consecutively across the group (a CTA finds
// its tensor by binary search over the start indices, which travel in the
// kernel parameters with the descriptors).  Each tensor keeps its own amax and
// scale; the per-CTA work is that of k_tensor_amax and k_tensor_cast, and the
// cast pass again takes the chunks last-to-first.
constexpr int kCurGroupMax = 128;  // tensors per launch (a 6.2 KiB parameter block)

struct CurTable {
    int count;
    int64_t start[kCurGroupMax + 1];
    CurrentTensor e[kCurGroupMax];
};
static_assert(sizeof(CurTable) <= 16384, "the grouped parameter block must stay well inside 32 KiB");

__device__ __forceinline__ int find_tensor(const CurTable& tab, int64_t b) {
    int lo = 0, hi = tab.count;  // start[lo] <= b < start[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tab.start[mid] <= b) lo = mid;
        else hi = mid;
    }
    return lo;
}

__global__ void k_zero_group_amax(const __grid_constant__ CurTable tab) {
    pdl_enter();
    for (int i = threadIdx.x; i < tab.count; i += blockDim.x) *tab.e[i].amax_out = 0.0f;
}

template <typename T, int BYTES>
__global__ void __launch_bounds__(kThreads) k_tensor_amax_grouped(const __grid_constant__ CurTable tab) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    const int t = find_tensor(tab, blockIdx.x);
    const CurrentTensor& e = tab.e[t];
    const int64_t nvec = e.n / V::kElems;
    const int tail_n = static_cast<int>(e.n - nvec * V::kElems);
    const int64_t chunk = static_cast<int64_t>(blockIdx.x) - tab.start[t];
    const auto* x = static_cast<const typename V::In*>(e.x);
    const int64_t base = chunk * kThreads * kUnroll + threadIdx.x;
    typename V::In v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        v[u] = (i < nvec) ? ld_words_stream(x + i) : V::zero();
    }
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) a = fmaxf(a, V::amax(v[u]));
    if (chunk == 0 && threadIdx.x < tail_n)
        a = fmaxf(a, fabsf(load_scalar(static_cast<const T*>(e.x) + nvec * V::kElems, threadIdx.x)));
    cta_amax_to_global(a, e.amax_out);
}

template <typename T, int FMT, int BYTES>
__global__ void __launch_bounds__(kThreads) k_tensor_cast_grouped(const __grid_constant__ CurTable tab) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    const int64_t b = tab.start[tab.count] - 1 - blockIdx.x;  // last-to-first
    const int t = find_tensor(tab, b);
    const CurrentTensor& e = tab.e[t];
    const int64_t nvec = e.n / V::kElems;
    const int tail_n = static_cast<int>(e.n - nvec * V::kElems);
    const int64_t chunk = b - tab.start[t];
    const auto* x = static_cast<const typename V::In*>(e.x);
    auto* q = reinterpret_cast<typename V::Out*>(e.q);
    const int64_t base = chunk * kThreads * kUnroll + threadIdx.x;
    typename V::In v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        v[u] = (i < nvec) ? ld_words_stream(x + i) : V::zero();
    }
    const float s = scale_from_amax<FMT>(*e.amax_out);
    const uint64_t s2 = f32x2(s, s);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        if (i < nvec) st_stream(q + i, V::template cast<FMT>(v[u], s2));
    }
    if (chunk == 0 && threadIdx.x < tail_n) {
        const float xv = load_scalar(static_cast<const T*>(e.x) + nvec * V::kElems, threadIdx.x);
        e.q[nvec * V::kElems + threadIdx.x] = static_cast<uint8_t>(cvt_fp8x2<FMT>(__fmul_rn(xv, s), 0.0f) & 0xFFu);
    }
    if (chunk == 0 && threadIdx.x == 0) *e.scale_out = s;
}

// ---------------------------------------------------------------------------
// Per-tensor cast with a second, transposed output: q [R, C] (optional) and
// qt [C, R] with qt[c][r] = q[r][c] -- the copy a weight-gradient GEMM reads
// along the other dimension.  One CTA per 128x128 tile: the tile's codes go
// through shared memory so that both outputs are written row by row.
// DELAYED / WITH_AMAX as in k_tensor_cast.
//
// Full tiles with vector-friendly strides load one lane vector per slice, 16
// rows per warp, as the 128x128 block kernel does; the read-out transposes
// 4x4-byte blocks in registers (byte permutes), and each warp writes whole
// 128-byte qt row segments.  Edge tiles and other strides take an
// element-wise path.  With current scaling the CTAs take the tiles
// last-to-first, so the first reads find the end of x that the amax pass
// left in L2.
// ---------------------------------------------------------------------------
// Resident CTAs per SM the transposing cast is compiled for (register cap):
// each CTA keeps one 32 KiB input tile in flight.
#ifndef FP8Q_TRANSPOSE_MIN_CTAS
#define FP8Q_TRANSPOSE_MIN_CTAS 4
#endif

template <typename T, int FMT, int BYTES, bool DELAYED, bool WITH_AMAX>
__global__ void __launch_bounds__(kThreads, FP8Q_TRANSPOSE_MIN_CTAS)
k_tensor_cast_transpose(const T* __restrict__ x, int64_t rows, int64_t cols, const float* scale_in,
                        const float* __restrict__ amax_in, uint8_t* __restrict__ q, uint8_t* __restrict__ qt,
                        float* scale_out, float* __restrict__ amax_out, int vector_ok) {
    pdl_enter();
    using V = LaneVec<T, BYTES>;
    __shared__ __align__(16) uint8_t tile[kTT * kTT];
    const int64_t tiles_c = (cols + kTT - 1) / kTT;
    const int64_t t = DELAYED ? blockIdx.x : gridDim.x - 1 - blockIdx.x;
    const int64_t tr = t / tiles_c;
    const int64_t tc = t - tr * tiles_c;
    const int64_t r0 = tr * kTT, c0 = tc * kTT;
    const int h = static_cast<int>(min(static_cast<int64_t>(kTT), rows - r0));
    const int w = static_cast<int>(min(static_cast<int64_t>(kTT), cols - c0));
    const float s = DELAYED ? *scale_in : scale_from_amax<FMT>(*amax_in);
    const uint64_t s2 = f32x2(s, s);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float a = 0.0f;

    if (vector_ok && h == kTT && w == kTT) {
        using G = TileGeom<T, BYTES>;
        const int lr0 = warp * 16 + lane / G::kVecPerRow, vec_in_row = lane % G::kVecPerRow;
        const auto* xv = reinterpret_cast<const typename V::In*>(x + (r0 + lr0) * cols + c0) + vec_in_row;
        const int64_t vstride = cols / V::kElems * G::kRowsPerLoad;  // lane vectors between this lane's rows
        typename V::In v[G::kLoads];
#pragma unroll
        for (int i = 0; i < G::kLoads; ++i) v[i] = ld_words_stream(xv + i * vstride);
        tile_cast<T, FMT, BYTES, WITH_AMAX>(v, s2, q, cols, r0, c0, tile, lr0, vec_in_row, a);
        __syncthreads();
        tile_transpose_out(tile, qt, rows, r0, c0, lane, warp);
    } else {
        for (int i = threadIdx.x; i < kTT * kTT; i += kThreads) {
            const int r = i / kTT, c = i % kTT;
            if (r < h && c < w) {
                const float xv = load_scalar(x + (r0 + r) * cols + c0, c);
                if (WITH_AMAX) a = fmaxf(a, fabsf(xv));
                const uint8_t code = static_cast<uint8_t>(cvt_fp8x2<FMT>(__fmul_rn(xv, s), 0.0f) & 0xFFu);
                if (q != nullptr) q[(r0 + r) * cols + c0 + c] = code;
                tile[tile_off(r, c)] = code;
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < kTT * kTT; i += kThreads) {
            const int c = i / kTT, r = i % kTT;
            if (r < h && c < w) qt[(c0 + c) * rows + r0 + r] = tile[tile_off(r, c)];
        }
    }
    if (WITH_AMAX) cta_amax_to_global(a, amax_out);
    if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = s;
}

// Zeroes the amax accumulator before the amax pass.  A kernel rather than a
// memset, so that the call's launches stay one programmatic-dependent-launch
// chain (a memset node would make the amax pass wait for a full completion).
__global__ void k_zero_f32(float* p) {
    pdl_enter();
    *p = 0.0f;
}

template <int FMT>
__global__ void k_scale_from_amax(const float* amax_in, float* scale_out) {
    pdl_enter();
    *scale_out = scale_from_amax<FMT>(*amax_in);
}

int64_t chunk_grid(int64_t nvec) {
    const int64_t per_cta = static_cast<int64_t>(kThreads) * kUnroll;
    return std::max<int64_t>(1, (nvec + per_cta - 1) / per_cta);
}

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <typename T, int BYTES>
cudaError_t amax_typed(const void* x, int64_t n, float* amax_out, cudaStream_t st) {
    using V = LaneVec<T, BYTES>;
    const int64_t nvec = n / V::kElems;
    const int tail_n = static_cast<int>(n - nvec * V::kElems);
    const T* tail = static_cast<const T*>(x) + nvec * V::kElems;
    auto kern = k_tensor_amax<T, BYTES>;
    const int64_t grid = chunk_grid(nvec);
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    {
        const cudaError_t e_ = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), 0, st, static_cast<const typename V::In*>(x), nvec, tail,
                                                           tail_n, amax_out);
        if (e_ != cudaSuccess) return e_;
    }
    return cudaGetLastError();
}

template <typename T, int FMT, int BYTES, bool DELAYED, bool WITH_AMAX>
cudaError_t cast_typed(const void* x, int64_t n, const float* scale_in, const float* amax_in, uint8_t* q,
                       float* scale_out, float* amax_out, cudaStream_t st) {
    using V = LaneVec<T, BYTES>;
    const int64_t nvec = n / V::kElems;
    const int tail_n = static_cast<int>(n - nvec * V::kElems);
    const T* tail = static_cast<const T*>(x) + nvec * V::kElems;
    auto kern = k_tensor_cast<T, FMT, BYTES, DELAYED, WITH_AMAX>;
    const int64_t grid = chunk_grid(nvec);
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    {
        const cudaError_t e_ = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), 0, st, static_cast<const typename V::In*>(x), nvec, tail, tail_n, scale_in, amax_in,
        reinterpret_cast<typename V::Out*>(q), q + nvec * V::kElems, scale_out, amax_out);
        if (e_ != cudaSuccess) return e_;
    }
    return cudaGetLastError();
}

template <typename T, int FMT, int BYTES>
cudaError_t cast_dispatch(const void* x, int64_t n, const float* scale_in, const float* amax_in, uint8_t* q,
                          float* scale_out, float* amax_out, cudaStream_t st) {
    if (scale_in == nullptr)
        return cast_typed<T, FMT, BYTES, false, false>(x, n, nullptr, amax_in, q, scale_out, nullptr, st);
    if (amax_out != nullptr)
        return cast_typed<T, FMT, BYTES, true, true>(x, n, scale_in, nullptr, q, scale_out, amax_out, st);
    return cast_typed<T, FMT, BYTES, true, false>(x, n, scale_in, nullptr, q, scale_out, nullptr, st);
}

template <typename T, int FMT>
cudaError_t cast_width(const void* x, int64_t n, const float* scale_in, const float* amax_in, uint8_t* q,
                       float* scale_out, float* amax_out, cudaStream_t st) {
    if (aligned32(x)) return cast_dispatch<T, FMT, 32>(x, n, scale_in, amax_in, q, scale_out, amax_out, st);
    return cast_dispatch<T, FMT, 16>(x, n, scale_in, amax_in, q, scale_out, amax_out, st);
}

template <typename T, int FMT, int BYTES, bool DELAYED, bool WITH_AMAX>
cudaError_t cast_transpose_typed(const void* x, int64_t rows, int64_t cols, const float* scale_in,
                                 const float* amax_in, uint8_t* q, uint8_t* qt, float* scale_out, float* amax_out,
                                 int vector_ok, cudaStream_t st) {
    const int64_t tiles = ((rows + kTT - 1) / kTT) * ((cols + kTT - 1) / kTT);
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const cudaError_t e = launch_kernel(k_tensor_cast_transpose<T, FMT, BYTES, DELAYED, WITH_AMAX>,
                                        dim3(static_cast<unsigned>(tiles)), dim3(kThreads), 0, st,
                                        static_cast<const T*>(x), rows, cols, scale_in, amax_in, q, qt, scale_out,
                                        amax_out, vector_ok);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename T, int FMT, int BYTES>
cudaError_t cast_transpose_mode(const void* x, int64_t rows, int64_t cols, const float* scale_in,
                                const float* amax_in, uint8_t* q, uint8_t* qt, float* scale_out, float* amax_out,
                                int vector_ok, cudaStream_t st) {
    if (scale_in == nullptr)
        return cast_transpose_typed<T, FMT, BYTES, false, false>(x, rows, cols, nullptr, amax_in, q, qt, scale_out,
                                                                 nullptr, vector_ok, st);
    if (amax_out != nullptr)
        return cast_transpose_typed<T, FMT, BYTES, true, true>(x, rows, cols, scale_in, nullptr, q, qt, scale_out,
                                                               amax_out, vector_ok, st);
    return cast_transpose_typed<T, FMT, BYTES, true, false>(x, rows, cols, scale_in, nullptr, q, qt, scale_out,
                                                            nullptr, vector_ok, st);
}

template <typename T, int FMT>
cudaError_t cast_transpose_width(const void* x, int64_t rows, int64_t cols, const float* scale_in,
                                 const float* amax_in, uint8_t* q, uint8_t* qt, float* scale_out, float* amax_out,
                                 cudaStream_t st) {
    // Vector path: every tile row starts on a 32-byte (else 16-byte) boundary
    // of x and a 16-byte boundary of q, and every qt run of 32 codes on a
    // 16-byte boundary.
    const int64_t rb = cols * static_cast<int64_t>(sizeof(T));
    const bool ok16 = (rb % 16 == 0) && (cols % 16 == 0) && (rows % 16 == 0);
    if (ok16 && aligned32(x) && rb % 32 == 0)
        return cast_transpose_mode<T, FMT, 32>(x, rows, cols, scale_in, amax_in, q, qt, scale_out, amax_out, 1, st);
    return cast_transpose_mode<T, FMT, 16>(x, rows, cols, scale_in, amax_in, q, qt, scale_out, amax_out,
                                           ok16 ? 1 : 0, st);
}

template <typename T, int FMT, int BYTES>
cudaError_t delayed_step_typed(const void* x, int64_t n, float* scale, uint8_t* q, float* scale_used,
                               float* amax_out, float* history, int32_t* state, int window, int algo, float alpha,
                               float margin, void* workspace, cudaStream_t st) {
    using V = LaneVec<T, BYTES>;
    const int64_t nvec = n / V::kElems;
    const int tail_n = static_cast<int>(n - nvec * V::kElems);
    const T* tail = static_cast<const T*>(x) + nvec * V::kElems;
    const int64_t grid = chunk_grid(nvec);
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const cudaError_t e = launch_kernel(k_tensor_cast_delayed_step<T, FMT, BYTES>, dim3(static_cast<unsigned>(grid)),
                                        dim3(kThreads), 0, st, static_cast<const typename V::In*>(x), nvec, tail,
                                        tail_n, scale, reinterpret_cast<typename V::Out*>(q), q + nvec * V::kElems,
                                        scale_used, amax_out, history, state, window, algo, alpha, margin,
                                        static_cast<StepWorkspace*>(workspace));
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t delayed_step_width(const void* x, int64_t n, float* scale, uint8_t* q, float* scale_used,
                               float* amax_out, float* history, int32_t* state, int window, int algo, float alpha,
                               float margin, void* workspace, cudaStream_t st) {
    if (aligned32(x))
        return delayed_step_typed<T, FMT, 32>(x, n, scale, q, scale_used, amax_out, history, state, window, algo,
                                              alpha, margin, workspace, st);
    return delayed_step_typed<T, FMT, 16>(x, n, scale, q, scale_used, amax_out, history, state, window, algo, alpha,
                                          margin, workspace, st);
}

}  // namespace

cudaError_t launch_tensor_delayed_step(const void* x, int dtype, int64_t n, int fmt, float* scale, uint8_t* q,
                                       float* scale_used, float* amax_out, float* history, int32_t* state,
                                       int window, int algo, float alpha, float margin, void* workspace,
                                       cudaStream_t st) {
    if (dtype == 1) {
        return fmt == kE4M3 ? delayed_step_width<uint16_t, kE4M3>(x, n, scale, q, scale_used, amax_out, history,
                                                                  state, window, algo, alpha, margin, workspace, st)
                            : delayed_step_width<uint16_t, kE5M2>(x, n, scale, q, scale_used, amax_out, history,
                                                                  state, window, algo, alpha, margin, workspace, st);
    }
    return fmt == kE4M3 ? delayed_step_width<float, kE4M3>(x, n, scale, q, scale_used, amax_out, history, state,
                                                           window, algo, alpha, margin, workspace, st)
                        : delayed_step_width<float, kE5M2>(x, n, scale, q, scale_used, amax_out, history, state,
                                                           window, algo, alpha, margin, workspace, st);
}

namespace {

template <typename T, int FMT, int BYTES>
cudaError_t delayed_grouped_typed(const DelayedTensor* t, int count, int window, int algo, float alpha, float margin,
                                  void* workspace, cudaStream_t st) {
    using V = LaneVec<T, BYTES>;
    StepTable tab;
    tab.window = window;
    tab.algo = algo;
    tab.alpha = alpha;
    tab.margin = margin;
    for (int first = 0; first < count; first += kStepGroupMax) {
        tab.count = std::min(kStepGroupMax, count - first);
        tab.ws = static_cast<StepWorkspace*>(workspace) + first;
        int64_t units = 0;
        for (int i = 0; i < tab.count; ++i) {
            tab.e[i] = t[first + i];
            tab.start[i] = units;
            units += chunk_grid(t[first + i].n / V::kElems);  // at least 1: the update runs for empty tensors
        }
        tab.start[tab.count] = units;
        if (units > 0x7FFFFFFF) return cudaErrorInvalidValue;
        const cudaError_t e = launch_kernel(k_tensor_cast_delayed_step_grouped<T, FMT, BYTES>,
                                            dim3(static_cast<unsigned>(units)), dim3(kThreads), 0, st, tab);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t delayed_grouped_width(const DelayedTensor* t, int count, int window, int algo, float alpha, float margin,
                                  void* workspace, cudaStream_t st) {
    bool w32 = true;  // 256-bit lanes only when every tensor allows them
    for (int i = 0; i < count; ++i) w32 = w32 && aligned32(t[i].x);
    return w32 ? delayed_grouped_typed<T, FMT, 32>(t, count, window, algo, alpha, margin, workspace, st)
               : delayed_grouped_typed<T, FMT, 16>(t, count, window, algo, alpha, margin, workspace, st);
}

}  // namespace

cudaError_t launch_tensor_delayed_step_grouped(const DelayedTensor* t, int count, int dtype, int fmt, int window,
                                               int algo, float alpha, float margin, void* workspace,
                                               cudaStream_t st) {
    if (dtype == 1)
        return fmt == kE4M3
                   ? delayed_grouped_width<uint16_t, kE4M3>(t, count, window, algo, alpha, margin, workspace, st)
                   : delayed_grouped_width<uint16_t, kE5M2>(t, count, window, algo, alpha, margin, workspace, st);
    return fmt == kE4M3 ? delayed_grouped_width<float, kE4M3>(t, count, window, algo, alpha, margin, workspace, st)
                        : delayed_grouped_width<float, kE5M2>(t, count, window, algo, alpha, margin, workspace, st);
}

namespace {

template <typename T, int FMT, int BYTES>
cudaError_t current_grouped_typed(const CurrentTensor* t, int count, cudaStream_t st) {
    using V = LaneVec<T, BYTES>;
    CurTable tab;
    for (int first = 0; first < count; first += kCurGroupMax) {
        tab.count = std::min(kCurGroupMax, count - first);
        int64_t units = 0;
        for (int i = 0; i < tab.count; ++i) {
            tab.e[i] = t[first + i];
            tab.start[i] = units;
            units += chunk_grid(t[first + i].n / V::kElems);  // at least 1: every tensor's scale is written
        }
        tab.start[tab.count] = units;
        if (units > 0x7FFFFFFF) return cudaErrorInvalidValue;
        cudaError_t e = launch_kernel(k_zero_group_amax, dim3(1), dim3(kCurGroupMax), 0, st, tab);
        if (e != cudaSuccess) return e;
        e = launch_kernel(k_tensor_amax_grouped<T, BYTES>, dim3(static_cast<unsigned>(units)), dim3(kThreads), 0, st,
                          tab);
        if (e != cudaSuccess) return e;
        e = launch_kernel(k_tensor_cast_grouped<T, FMT, BYTES>, dim3(static_cast<unsigned>(units)), dim3(kThreads),
                          0, st, tab);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

template <typename T, int FMT>
cudaError_t current_grouped_width(const CurrentTensor* t, int count, cudaStream_t st) {
    bool w32 = true;  // 256-bit lanes only when every tensor allows them
    for (int i = 0; i < count; ++i) w32 = w32 && aligned32(t[i].x);
    return w32 ? current_grouped_typed<T, FMT, 32>(t, count, st) : current_grouped_typed<T, FMT, 16>(t, count, st);
}

}  // namespace

cudaError_t launch_tensor_current_grouped(const CurrentTensor* t, int count, int dtype, int fmt, cudaStream_t st) {
    if (count <= 0) return cudaSuccess;
    if (dtype == 1)
        return fmt == kE4M3 ? current_grouped_width<uint16_t, kE4M3>(t, count, st)
                            : current_grouped_width<uint16_t, kE5M2>(t, count, st);
    return fmt == kE4M3 ? current_grouped_width<float, kE4M3>(t, count, st)
                        : current_grouped_width<float, kE5M2>(t, count, st);
}

cudaError_t launch_tensor_cast_transpose(const void* x, int dtype, int64_t rows, int64_t cols, int fmt,
                                         const float* scale_in, const float* amax_in, uint8_t* q, uint8_t* qt,
                                         float* scale_out, float* amax_out, cudaStream_t st) {
    if (dtype == 1) {
        return fmt == kE4M3
                   ? cast_transpose_width<uint16_t, kE4M3>(x, rows, cols, scale_in, amax_in, q, qt, scale_out, amax_out, st)
                   : cast_transpose_width<uint16_t, kE5M2>(x, rows, cols, scale_in, amax_in, q, qt, scale_out, amax_out, st);
    }
    return fmt == kE4M3
               ? cast_transpose_width<float, kE4M3>(x, rows, cols, scale_in, amax_in, q, qt, scale_out, amax_out, st)
               : cast_transpose_width<float, kE5M2>(x, rows, cols, scale_in, amax_in, q, qt, scale_out, amax_out, st);
}

cudaError_t launch_tensor_amax(const void* x, int dtype, int64_t n, float* amax_out, cudaStream_t st) {
    if (dtype == 1)
        return aligned32(x) ? amax_typed<uint16_t, 32>(x, n, amax_out, st) : amax_typed<uint16_t, 16>(x, n, amax_out, st);
    return aligned32(x) ? amax_typed<float, 32>(x, n, amax_out, st) : amax_typed<float, 16>(x, n, amax_out, st);
}

cudaError_t launch_zero_f32(float* p, cudaStream_t st) {
    return launch_kernel(k_zero_f32, dim3(1), dim3(1), 0, st, p);
}

cudaError_t launch_scale_from_amax(const float* amax_in, int fmt, float* scale_out, cudaStream_t st) {
    if (fmt == kE4M3) return launch_kernel(k_scale_from_amax<kE4M3>, dim3(1), dim3(1), 0, st, amax_in, scale_out);
    return launch_kernel(k_scale_from_amax<kE5M2>, dim3(1), dim3(1), 0, st, amax_in, scale_out);
}

cudaError_t launch_tensor_cast(const void* x, int dtype, int64_t n, int fmt, const float* scale_in,
                               const float* amax_in, uint8_t* q, float* scale_out, float* amax_out,
                               cudaStream_t st) {
    if (dtype == 1) {
        return fmt == kE4M3 ? cast_width<uint16_t, kE4M3>(x, n, scale_in, amax_in, q, scale_out, amax_out, st)
                            : cast_width<uint16_t, kE5M2>(x, n, scale_in, amax_in, q, scale_out, amax_out, st);
    }
    return fmt == kE4M3 ? cast_width<float, kE4M3>(x, n, scale_in, amax_in, q, scale_out, amax_out, st)
                        : cast_width<float, kE5M2>(x, n, scale_in, amax_in, q, scale_out, amax_out, st);
}

}  // namespace fp8q
