// history_update.cuh -- one step of delayed scaling, run by one warp.
//
// PyTorch-FP8 page s4.2 DelayedScaler.update and the s4.3 refinements:
//   algo 0: push amax into the ring of the last `window` amax values; once the
//           window is full, scale = MAX / RN(max(max(window), eps) * margin);
//   algo 1: exponential moving average m of amax in history[0] (the first
//           update sets m = amax, later ones m = RN(RN(alpha*amax) +
//           RN(RN(1-alpha)*m))); state[1] counts updates up to `window`, and
//           from then on every update sets scale = MAX / RN(max(m, eps) * margin).
// Used by the stand-alone update kernel and by the last CTA of the fused
// delayed-scaling cast.  Out-of-range state is brought into range instead of
// indexing outside the ring: pos modulo window, count clamped to [0, window].
#pragma once

#include <cstdint>

#include "fp8q_device.cuh"

namespace fp8q {

// MAX / (max(amax, eps) * margin), both operations rounded in fp32.
template <int FMT>
__device__ __forceinline__ float scale_with_margin(float amax, float margin) {
    return __fdiv_rn(fmt_max<FMT>(), __fmul_rn(fmaxf(amax, kAmaxEps), margin));
}

// Executed by all 32 lanes of one warp (a is the same in every lane).
template <int FMT>
__device__ __forceinline__ void history_update_warp(float* history, int32_t* state, int window, float a,
                                                    float* scale, int algo, float alpha, float margin) {
    const int lane = threadIdx.x & 31;
    int count = min(max(state[1], 0), window);
    if (algo == 1) {
        if (lane == 0) {
            const float m = (count == 0)
                ? a
                : __fadd_rn(__fmul_rn(alpha, a), __fmul_rn(__fsub_rn(1.0f, alpha), history[0]));
            history[0] = m;
            count = min(count + 1, window);
            state[1] = count;
            if (count == window) *scale = scale_with_margin<FMT>(m, margin);
        }
        return;
    }
    int pos = state[0] % window;
    if (pos < 0) pos += window;
    count = min(count + 1, window);
    // max over the window as it will be after this push: slot `pos` holds the
    // new amax.  fmaxf ignores a NaN operand.
    float m = 0.0f;
    for (int i = lane; i < window; i += 32) m = fmaxf(m, (i == pos) ? a : history[i]);
    m = warp_max<32>(m);
    __syncwarp();  // every lane has read history[] before lane 0 writes it
    if (lane == 0) {
        history[pos] = a;
        state[0] = (pos + 1 == window) ? 0 : pos + 1;
        state[1] = count;
        if (count == window) *scale = scale_with_margin<FMT>(m, margin);
    }
}

}  // namespace fp8q
