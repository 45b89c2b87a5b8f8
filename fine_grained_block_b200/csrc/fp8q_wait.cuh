// fp8q_wait.cuh -- bounded waits.
//
// No kernel here waits forever.  A wait gives up after a limit measured with
// the global nanosecond timer; the caller then records the wait-timeout bit in
// the library's device status word (fp8_device_status) and returns.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp8q {

// Device status bits, readable through fp8_device_status().
constexpr unsigned int kStatusWaitTimeout = 1u;

// Default limit for one wait: the grid-wide barrier of the one-pass kernel
// completes in microseconds, so a second means it never will.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned int ld_volatile_u32(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Spin until *word differs from `seen`; false if limit_ns passes first.
__device__ __forceinline__ bool wait_for_change(const unsigned int* word, unsigned int seen, uint64_t limit_ns) {
    if (ld_volatile_u32(word) != seen) return true;
    const uint64_t start = global_timer_ns();
    while (ld_volatile_u32(word) == seen) {
        if (global_timer_ns() - start > limit_ns) return false;
    }
    return true;
}

}  // namespace fp8q
