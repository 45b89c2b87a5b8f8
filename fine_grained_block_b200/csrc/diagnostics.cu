// diagnostics.cu -- the library's device status word.
//
// Kernels that wait (at the one-pass kernel's grid-wide barrier) never wait
// forever: a wait that runs out sets a bit here and the kernel returns.  The
// word lives in this file; other kernels receive its device address as an
// argument (device_status_word()), so no relocatable device code is needed.

#include <atomic>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "fp8q_wait.cuh"

namespace fp8q {
namespace {

__device__ unsigned int g_device_status = 0u;

__global__ void k_device_status(unsigned int* out, int clear) {
    out[0] = clear ? atomicExch(&g_device_status, 0u) : atomicOr(&g_device_status, 0u);
}

// A word that nothing ever changes: the same bounded wait the one-pass kernel
// uses at its grid barrier must give up on it.
__device__ unsigned int g_never_changes = 0u;

__global__ void k_selftest_wait_timeout(uint64_t limit_ns) {
    if (!wait_for_change(&g_never_changes, 0u, limit_ns)) atomicOr(&g_device_status, kStatusWaitTimeout);
}

}  // namespace

unsigned int* device_status_word() {
    static std::atomic<unsigned int*> cache[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
    unsigned int* p = cache[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_device_status) != cudaSuccess) return nullptr;
        p = static_cast<unsigned int*>(addr);
        cache[dev].store(p, std::memory_order_release);
    }
    return p;
}

cudaError_t launch_device_status(unsigned int* out, int clear, cudaStream_t st) {
    k_device_status<<<1, 1, 0, st>>>(out, clear);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t st) {
    k_selftest_wait_timeout<<<1, 1, 0, st>>>(limit_ns);
    return cudaGetLastError();
}

}  // namespace fp8q
