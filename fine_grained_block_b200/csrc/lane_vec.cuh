// lane_vec.cuh -- one lane's slice of a streaming kernel: a 16- or 32-byte
// vector of bf16 or fp32 inputs, its |x| maximum, and its scaled cast to FP8
// codes.  32-byte vectors use one 256-bit access per lane (sm_100); 16-byte
// vectors serve pointers that are only 16-byte aligned.
#pragma once

#include <cstdint>

#include "fp8q_device.cuh"

namespace fp8q {

template <int N>
struct Words {
    uint32_t w[N];
};

__device__ __forceinline__ Words<4> ld_words_stream(const Words<4>* p) {
    const uint4 v = ld_stream(reinterpret_cast<const uint4*>(p));
    return Words<4>{{v.x, v.y, v.z, v.w}};
}
__device__ __forceinline__ Words<8> ld_words_stream(const Words<8>* p) {
    const V32 v = ld32_stream(p);
    Words<8> r;
#pragma unroll
    for (int k = 0; k < 8; ++k) r.w[k] = v.w[k];
    return r;
}

// Codes of one lane: kCodeWords 32-bit words (4, 8 or 16 codes).
template <int NW>
struct CodeWords;
template <>
struct CodeWords<1> {
    using T = uint32_t;
    static __device__ __forceinline__ T make(const uint32_t* c) { return c[0]; }
};
template <>
struct CodeWords<2> {
    using T = uint2;
    static __device__ __forceinline__ T make(const uint32_t* c) { return make_uint2(c[0], c[1]); }
};
template <>
struct CodeWords<4> {
    using T = uint4;
    static __device__ __forceinline__ T make(const uint32_t* c) { return make_uint4(c[0], c[1], c[2], c[3]); }
};

template <typename T, int BYTES>
struct LaneVec;

// bf16 bit patterns: 2 elements per word.
template <int BYTES>
struct LaneVec<uint16_t, BYTES> {
    static constexpr int kWords = BYTES / 4;
    static constexpr int kElems = BYTES / 2;
    using In = Words<kWords>;
    using Out = typename CodeWords<kWords / 2>::T;

    static __device__ __forceinline__ In zero() {
        In v;
#pragma unroll
        for (int k = 0; k < kWords; ++k) v.w[k] = 0u;
        return v;
    }
    static __device__ __forceinline__ float amax(const In& v) {
        uint32_t m[kWords];
#pragma unroll
        for (int k = 0; k < kWords; ++k) m[k] = v.w[k];
#pragma unroll
        for (int width = kWords / 2; width > 0; width /= 2)
#pragma unroll
            for (int k = 0; k < width; ++k) m[k] = xabsmax_bf16x2(m[k], m[k + width]);
        return bf16x2_absmax_finish(m[0]);
    }
    template <int FMT>
    static __device__ __forceinline__ Out cast(const In& v, uint64_t s2) {
        uint32_t c[kWords / 2];
#pragma unroll
        for (int k = 0; k < kWords / 2; ++k)
            c[k] = scale_cast_bf16x2<FMT>(v.w[2 * k], s2) | (scale_cast_bf16x2<FMT>(v.w[2 * k + 1], s2) << 16);
        return CodeWords<kWords / 2>::make(c);
    }
};

// fp32: 1 element per word.
template <int BYTES>
struct LaneVec<float, BYTES> {
    static constexpr int kWords = BYTES / 4;
    static constexpr int kElems = BYTES / 4;
    using In = Words<kWords>;
    using Out = typename CodeWords<kWords / 4>::T;

    static __device__ __forceinline__ In zero() {
        In v;
#pragma unroll
        for (int k = 0; k < kWords; ++k) v.w[k] = 0u;
        return v;
    }
    static __device__ __forceinline__ float amax(const In& v) {
        float m = fabsf(__uint_as_float(v.w[0]));
#pragma unroll
        for (int k = 1; k < kWords; ++k) m = fmaxf(m, fabsf(__uint_as_float(v.w[k])));
        return m;
    }
    template <int FMT>
    static __device__ __forceinline__ Out cast(const In& v, uint64_t s2) {
        uint32_t c[kWords / 4];
#pragma unroll
        for (int k = 0; k < kWords / 4; ++k)
            c[k] = scale_cast_f32x2<FMT>(v.w[4 * k], v.w[4 * k + 1], s2) |
                   (scale_cast_f32x2<FMT>(v.w[4 * k + 2], v.w[4 * k + 3], s2) << 16);
        return CodeWords<kWords / 4>::make(c);
    }
};

}  // namespace fp8q
