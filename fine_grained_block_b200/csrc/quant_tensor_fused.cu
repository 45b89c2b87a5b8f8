// quant_tensor_fused.cu -- per-tensor current scaling in ONE pass over x, for
// tensors that fit in the registers of the CTAs that can be resident at once.
//
// PyTorch-FP8 page s4.1 (scale = max_val / amax) and mixed-precision handbook
// "FP8 training" per_tensor: the scale needs the amax of the whole tensor
// before any element is cast, which normally costs a second read of x.  Here
// every CTA loads its slice of x into registers, folds its amax into a small
// workspace, and waits at a grid-wide barrier; the last CTA to arrive writes
// amax_out and scale_out and resets the workspace; then every CTA casts the
// slice it still holds.  x is read once and the three launches of the
// two-pass path (zeroing, amax, cast) become one.
//
// The launch is cooperative, so all CTAs are co-resident and the barrier
// cannot deadlock.  The barrier wait is still bounded (about a second); if it
// runs out the CTA records the wait-timeout bit in the device status word and
// returns without writing its codes.
//
// Workspace (16 bytes of device memory, zero before the first use; every call
// leaves it ready for the next): {arrivals, amax bits, result}, where result
// packs the amax bits of the last completed call (low half) with the count of
// completed calls (high half).  Calls that share a workspace must not overlap
// on the device.
//
// The barrier keeps the chain of dependent global-memory trips short.  Each
// CTA reads the call count when it starts, while its loads of x are in
// flight.  At the barrier it folds its amax in (an atomic max, fenced) and
// arrives (an atomic add).  The last to arrive reads the final amax, writes
// amax_out and scale_out, clears the arrival count and the running amax, and
// publishes {amax, count + 1} in the result word with one 64-bit store.  The
// others spin on that word until its count moves on and take the amax from
// it, so they need no further read.

#include <algorithm>
#include <cstddef>
#include <atomic>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "fp8q_wait.cuh"
#include "lane_vec.cuh"

namespace fp8q {

namespace {

constexpr int kThreads = 256;
constexpr int kLoads = 4;  // lane vectors per thread held in registers

struct Workspace {
    unsigned int arrivals;        // CTAs of the current call that have arrived
    unsigned int amax_bits;       // running max of the current call's CTA maxima
    unsigned long long result;    // {amax bits of the last completed call, completed calls}
};
static_assert(sizeof(Workspace) == 16, "workspace layout");
static_assert(offsetof(Workspace, result) == 8, "the result word is 8-byte aligned in a 16-byte-aligned workspace");

__device__ __forceinline__ unsigned long long ld_volatile_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.volatile.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_volatile_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.volatile.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Spin until the call count in the result word differs from `count`; the word
// then holds the amax of this call.  False if limit_ns passes first.
__device__ __forceinline__ bool wait_for_result(const unsigned long long* word, unsigned int count,
                                                unsigned long long* out, uint64_t limit_ns) {
    unsigned long long r = ld_volatile_u64(word);
    if (static_cast<unsigned int>(r >> 32) != count) {
        *out = r;
        return true;
    }
    const uint64_t start = global_timer_ns();
    for (;;) {
        r = ld_volatile_u64(word);
        if (static_cast<unsigned int>(r >> 32) != count) {
            *out = r;
            return true;
        }
        if (global_timer_ns() - start > limit_ns) return false;
    }
}

template <typename T>
__device__ __forceinline__ float load_scalar(const T* p, int i);
template <>
__device__ __forceinline__ float load_scalar<uint16_t>(const uint16_t* p, int i) {
    return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
}
template <>
__device__ __forceinline__ float load_scalar<float>(const float* p, int i) { return p[i]; }

template <typename T, int FMT, int BYTES>
__global__ void __launch_bounds__(kThreads)
k_tensor_fused(const typename LaneVec<T, BYTES>::In* __restrict__ x, int64_t nvec, const T* __restrict__ tail,
               int tail_n, typename LaneVec<T, BYTES>::Out* __restrict__ q, uint8_t* __restrict__ q_tail,
               float* scale_out, float* amax_out, Workspace* ws, unsigned int* status) {
    using V = LaneVec<T, BYTES>;
    __shared__ float warp_amax[kThreads / 32];
    __shared__ float cta_result;
    __shared__ int cta_ok;

    // the call count, read while the loads below are in flight: it cannot move before this CTA arrives
    unsigned int count = 0;
    if (threadIdx.x == 0) count = static_cast<unsigned int>(ld_volatile_u64(&ws->result) >> 32);
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads * kLoads + threadIdx.x;
    typename V::In v[kLoads];
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
        const int64_t i = base + u * kThreads;
        v[u] = (i < nvec) ? ld_words_stream(x + i) : V::zero();
    }
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < kLoads; ++u) a = fmaxf(a, V::amax(v[u]));
    float xt = 0.0f;
    if (blockIdx.x == 0 && threadIdx.x < tail_n) {
        xt = load_scalar(tail, threadIdx.x);
        a = fmaxf(a, fabsf(xt));
    }
    a = warp_max<32>(a);
    if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = a;
    __syncthreads();

    if (threadIdx.x == 0) {
        float m = warp_amax[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, warp_amax[w]);
        // contribute this CTA's amax, then arrive: the arrival's release half orders the max before it,
        // and its acquire half makes every earlier arrival's max visible to the last CTA
        atomicMax(&ws->amax_bits, __float_as_uint(m));
        unsigned int arrived;
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(arrived) : "l"(&ws->arrivals) : "memory");
        bool ok = true;
        float amax;
        if (arrived == gridDim.x - 1) {
            // last to arrive: every other CTA's atomicMax was performed before its arrival
            const unsigned int bits = atomicOr(&ws->amax_bits, 0u);
            amax = __uint_as_float(bits);
            *amax_out = amax;
            *scale_out = scale_from_amax<FMT>(amax);
            ws->amax_bits = 0u;
            ws->arrivals = 0u;
            // the waiting CTAs read nothing but this word, so no fence is needed before it
            st_volatile_u64(&ws->result, (static_cast<unsigned long long>(count + 1u) << 32) | bits);
        } else {
            unsigned long long r = 0;
            ok = wait_for_result(&ws->result, count, &r, kWaitLimitNs);
            amax = __uint_as_float(static_cast<unsigned int>(r));
        }
        if (!ok) atomicOr(status, kStatusWaitTimeout);
        cta_result = amax;
        cta_ok = ok ? 1 : 0;
    }
    __syncthreads();
    if (!cta_ok) return;

    const float s = scale_from_amax<FMT>(cta_result);
    const uint64_t s2 = f32x2(s, s);
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
        const int64_t i = base + u * kThreads;
        if (i < nvec) st_stream(q + i, V::template cast<FMT>(v[u], s2));
    }
    if (blockIdx.x == 0 && threadIdx.x < tail_n)
        q_tail[threadIdx.x] = static_cast<uint8_t>(cvt_fp8x2<FMT>(__fmul_rn(xt, s), 0.0f) & 0xFFu);
}

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// Largest grid that can be co-resident, or -1 when it cannot be known: a failed
// CUDA query, or a device without cooperative launch.  A known answer is kept
// per device (one cache per kernel), so calls after the first make one CUDA
// call here (cudaGetDevice) instead of four.
template <typename Kernel>
int64_t resident_ctas(Kernel k) {
    static std::atomic<int64_t> cache[128];
    int dev = 0, coop = 0, per_sm = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (dev >= 0 && dev < 128) {
        const int64_t known = cache[dev].load(std::memory_order_acquire);
        if (known > 0) return known;
    }
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) return -1;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return -1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, 0) != cudaSuccess) return -1;
    const int64_t units = static_cast<int64_t>(per_sm) * sms;
    if (units > 0 && dev >= 0 && dev < 128) cache[dev].store(units, std::memory_order_release);
    return units;
}

template <typename T, int FMT, int BYTES>
cudaError_t fused_typed(const void* x, int64_t n, uint8_t* q, float* scale_out, float* amax_out, void* ws,
                        cudaStream_t st, bool* launched) {
    using V = LaneVec<T, BYTES>;
    auto kern = k_tensor_fused<T, FMT, BYTES>;
    const int64_t nvec = n / V::kElems;
    const int tail_n = static_cast<int>(n - nvec * V::kElems);
    const int64_t per_cta = static_cast<int64_t>(kThreads) * kLoads;
    const int64_t grid = std::max<int64_t>(1, (nvec + per_cta - 1) / per_cta);
    *launched = false;
    const int64_t resident = resident_ctas(kern);
    if (resident < 0 || grid > resident) return cudaSuccess;  // unknown or too large for one pass: caller falls back
    const typename V::In* xv = static_cast<const typename V::In*>(x);
    const T* tail = static_cast<const T*>(x) + nvec * V::kElems;
    typename V::Out* qv = reinterpret_cast<typename V::Out*>(q);
    uint8_t* q_tail = q + nvec * V::kElems;
    Workspace* w = static_cast<Workspace*>(ws);
    unsigned int* status = device_status_word();
    if (status == nullptr) return cudaErrorInvalidValue;
    int64_t nvec_arg = nvec;
    int tail_arg = tail_n;
    void* args[] = {&xv, &nvec_arg, &tail, &tail_arg, &qv, &q_tail, &scale_out, &amax_out, &w, &status};
    cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(static_cast<unsigned>(grid)),
                                                dim3(kThreads), args, 0, st);
    if (e == cudaSuccess) *launched = true;
    return e;
}

template <typename T, int FMT>
cudaError_t fused_width(const void* x, int64_t n, uint8_t* q, float* scale_out, float* amax_out, void* ws,
                        cudaStream_t st, bool* launched) {
    if (aligned32(x)) return fused_typed<T, FMT, 32>(x, n, q, scale_out, amax_out, ws, st, launched);
    return fused_typed<T, FMT, 16>(x, n, q, scale_out, amax_out, ws, st, launched);
}

// 1: n elements fit one pass; 0: they do not; -1: the co-resident grid cannot be known.
template <typename T, int FMT, int BYTES>
int fused_fit_typed(int64_t n) {
    using V = LaneVec<T, BYTES>;
    const int64_t per_cta = static_cast<int64_t>(kThreads) * kLoads;
    const int64_t grid = std::max<int64_t>(1, (n / V::kElems + per_cta - 1) / per_cta);
    const int64_t resident = resident_ctas(k_tensor_fused<T, FMT, BYTES>);
    if (resident < 0) return -1;
    return grid <= resident ? 1 : 0;
}

// ---------------------------------------------------------------------------
// Scratch for callers that cannot allocate device memory: a fixed array in
// this module's device memory, which every GPU that loads the library keeps
// until the process exits.  Its maximum size is kNoAllocScratchBytes; the
// one-pass kernel uses the first sizeof(Workspace) bytes of it as its
// workspace.  Host code cannot use the array's name as a device address, so
// the address is looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = 256;
static_assert(sizeof(Workspace) <= kNoAllocScratchBytes, "the workspace must fit the fixed scratch");
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch for the current device (looked up on
// the first call on that device and cached for the life of the process), or
// nullptr if the lookup failed.  The cache does not survive cudaDeviceReset:
// after a reset the module is loaded again and the array may move.
void* noalloc_scratch_address() {
    static std::atomic<void*> cache[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
    void* p = cache[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
        cache[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

int tensor_fused_fit(const void* x, int dtype, int64_t n, int fmt) {
    const bool w32 = aligned32(x);
    if (dtype == 1) {
        if (fmt == kE4M3) return w32 ? fused_fit_typed<uint16_t, kE4M3, 32>(n) : fused_fit_typed<uint16_t, kE4M3, 16>(n);
        return w32 ? fused_fit_typed<uint16_t, kE5M2, 32>(n) : fused_fit_typed<uint16_t, kE5M2, 16>(n);
    }
    if (fmt == kE4M3) return w32 ? fused_fit_typed<float, kE4M3, 32>(n) : fused_fit_typed<float, kE4M3, 16>(n);
    return w32 ? fused_fit_typed<float, kE5M2, 32>(n) : fused_fit_typed<float, kE5M2, 16>(n);
}

cudaError_t launch_tensor_fused_noalloc(const void* x, int dtype, int64_t n, int fmt, uint8_t* q, float* scale_out,
                                        float* amax_out, cudaStream_t st) {
    void* ws = noalloc_scratch_address();
    if (ws == nullptr) return cudaErrorInvalidSymbol;
    // The array keeps whatever the last call left; the workspace must start at zero.
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(Workspace), st);
    if (e != cudaSuccess) return e;
    bool launched = false;
    e = launch_tensor_fused(x, dtype, n, fmt, q, scale_out, amax_out, ws, st, &launched);
    if (e == cudaSuccess && !launched) return cudaErrorInvalidValue;  // the caller checks the size first
    return e;
}

cudaError_t launch_tensor_fused(const void* x, int dtype, int64_t n, int fmt, uint8_t* q, float* scale_out,
                                float* amax_out, void* workspace, cudaStream_t st, bool* launched) {
    if (dtype == 1) {
        return fmt == kE4M3 ? fused_width<uint16_t, kE4M3>(x, n, q, scale_out, amax_out, workspace, st, launched)
                            : fused_width<uint16_t, kE5M2>(x, n, q, scale_out, amax_out, workspace, st, launched);
    }
    return fmt == kE4M3 ? fused_width<float, kE4M3>(x, n, q, scale_out, amax_out, workspace, st, launched)
                        : fused_width<float, kE5M2>(x, n, q, scale_out, amax_out, workspace, st, launched);
}

}  // namespace fp8q
