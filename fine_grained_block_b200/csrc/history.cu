// history.cu -- delayed scaling: the amax history and the scale it yields.
//
// PyTorch-FP8 page, s4.2 DelayedScaler: keep the amax of the last `window`
// steps; once the window is full, scale = max_val / max(max(window), eps).
// The scale used by step k therefore comes from steps k-window .. k-1, which
// is what lets the cast run without a global reduction first (s4.1, s4.2).
//
// The ring buffer, its {pos, count} state and the scale live in device memory,
// so a training loop runs quantize -> update -> quantize ... with no host
// round trip.

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "history_update.cuh"
#include "launch_util.h"

namespace fp8q {
namespace {

template <int FMT>
__global__ void __launch_bounds__(32)
k_amax_history_update(float* __restrict__ history, int32_t* __restrict__ state, int window,
                      const float* __restrict__ amax, float* __restrict__ scale) {
    pdl_enter();
    const int lane = threadIdx.x;
    // Out-of-range state is brought into range instead of indexing outside
    // the ring: pos modulo window, count clamped to [0, window].
    int pos = state[0] % window;
    if (pos < 0) pos += window;
    int count = min(max(state[1], 0), window);
    const float a = *amax;
    count = min(count + 1, window);
    // Max over the window as it will be after this push: slot `pos` holds the
    // new amax.  fmaxf ignores a NaN operand.
    float m = 0.0f;
    for (int i = lane; i < window; i += 32) m = fmaxf(m, (i == pos) ? a : history[i]);
    m = warp_max<32>(m);
    __syncwarp();  // every lane has read history[] before lane 0 writes it
    if (lane == 0) {
        history[pos] = a;
        state[0] = (pos + 1 == window) ? 0 : pos + 1;
        state[1] = count;
        if (count == window) *scale = scale_from_amax<FMT>(m);
    }
}

template <int FMT>
__global__ void __launch_bounds__(32)
k_amax_history_update_ex(float* __restrict__ history, int32_t* __restrict__ state, int window,
                         const float* __restrict__ amax, float* __restrict__ scale, int algo, float alpha,
                         float margin) {
    pdl_enter();
    history_update_warp<FMT>(history, state, window, *amax, scale, algo, alpha, margin);
}

}  // namespace

cudaError_t launch_amax_history_update_ex(float* history, int32_t* state, int window, const float* amax, int fmt,
                                          float* scale, int algo, float alpha, float margin, cudaStream_t st) {
    if (fmt == kE4M3)
        return launch_kernel(k_amax_history_update_ex<kE4M3>, dim3(1), dim3(32), 0, st, history, state, window, amax,
                             scale, algo, alpha, margin);
    return launch_kernel(k_amax_history_update_ex<kE5M2>, dim3(1), dim3(32), 0, st, history, state, window, amax,
                         scale, algo, alpha, margin);
}

cudaError_t launch_amax_history_update(float* history, int32_t* state, int window, const float* amax, int fmt,
                                       float* scale, cudaStream_t st) {
    if (fmt == kE4M3)
        return launch_kernel(k_amax_history_update<kE4M3>, dim3(1), dim3(32), 0, st, history, state, window, amax, scale);
    return launch_kernel(k_amax_history_update<kE5M2>, dim3(1), dim3(32), 0, st, history, state, window, amax, scale);
}

}  // namespace fp8q
