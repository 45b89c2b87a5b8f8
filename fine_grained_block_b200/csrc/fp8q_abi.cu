// fp8q_abi.cu -- the C ABI of libfp8q (declared in include/fp8q.h).
//
// Each entry point checks every argument on the host, then enqueues its
// kernels on the caller's stream and returns.  Nothing here allocates,
// synchronizes or keeps state between calls, apart from a per-device cache of
// the SM count.

#include <atomic>
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "fp8q.h"
#include "fp8q_launch.h"


namespace fp8q {

int device_sm_count() {
    static std::atomic<int> cache[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

}  // namespace fp8q

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool fmt_ok(int fmt) { return fmt == FP8_E4M3 || fmt == FP8_E5M2; }
bool dtype_ok(int dt) { return dt == FP8_F32 || dt == FP8_BF16; }

// rows * cols without overflow (both >= 0); -1 if it would overflow.
int64_t checked_count(int64_t rows, int64_t cols) {
    if (rows == 0 || cols == 0) return 0;
    if (rows > INT64_MAX / cols) return -1;
    return rows * cols;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA; }

}  // namespace

extern "C" {

int fp8_quantize_per_tensor(const void* x, int dtype, int64_t n, int fmt, const float* scale_in, uint8_t* q,
                            float* scale_out, float* amax_out, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (scale_out == nullptr) return FP8_ERR_NULL;
    if (scale_in == nullptr && amax_out == nullptr) return FP8_ERR_NULL;
    if (n > 0 && (x == nullptr || q == nullptr)) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale_out, 4) || !aligned(scale_in, 4) ||
        !aligned(amax_out, 4))
        return FP8_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (amax_out != nullptr) {
        cudaError_t e = fp8q::launch_zero_f32(amax_out, st);
        if (e != cudaSuccess) return FP8_ERR_CUDA;
    }
    if (scale_in == nullptr && n > 0) {
        cudaError_t e = fp8q::launch_tensor_amax(x, dtype, n, amax_out, st);
        if (e != cudaSuccess) return FP8_ERR_CUDA;
    }
    return status_of(fp8q::launch_tensor_cast(x, dtype, n, fmt, scale_in, amax_out, q, scale_out,
                                              scale_in ? amax_out : nullptr, st));
}

int fp8_quantize_per_tensor_fused(const void* x, int dtype, int64_t n, int fmt, uint8_t* q, float* scale_out,
                                  float* amax_out, void* workspace, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (scale_out == nullptr || amax_out == nullptr || workspace == nullptr) return FP8_ERR_NULL;
    if (n > 0 && (x == nullptr || q == nullptr)) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale_out, 4) || !aligned(amax_out, 4) ||
        !aligned(workspace, 16))
        return FP8_ERR_ALIGN;
    if (n > 0) {
        bool launched = false;
        const cudaError_t e = fp8q::launch_tensor_fused(x, dtype, n, fmt, q, scale_out, amax_out, workspace,
                                                        static_cast<cudaStream_t>(stream), &launched);
        if (e != cudaSuccess) return FP8_ERR_CUDA;
        if (launched) return FP8_OK;
    }
    return fp8_quantize_per_tensor(x, dtype, n, fmt, nullptr, q, scale_out, amax_out, stream);
}

int fp8_quantize_per_tensor_fused_noalloc(const void* x, int dtype, int64_t n, int fmt, uint8_t* q, float* scale_out,
                                          float* amax_out, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (scale_out == nullptr || amax_out == nullptr) return FP8_ERR_NULL;
    if (n > 0 && (x == nullptr || q == nullptr)) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale_out, 4) || !aligned(amax_out, 4)) return FP8_ERR_ALIGN;
    if (n == 0) return fp8_quantize_per_tensor(x, dtype, n, fmt, nullptr, q, scale_out, amax_out, stream);
    const int fit = fp8q::tensor_fused_fit(x, dtype, n, fmt);
    if (fit < 0) return FP8_ERR_CUDA;  // the capacity cannot be known on this device
    if (fit == 0) return FP8_ERR_TOO_LARGE;
    return status_of(fp8q::launch_tensor_fused_noalloc(x, dtype, n, fmt, q, scale_out, amax_out,
                                                       static_cast<cudaStream_t>(stream)));
}

int fp8_quantize_blockwise_transpose(const void* x, int dtype, int64_t rows, int64_t cols, int block_rows,
                                     int block_cols, int fmt, uint8_t* q, float* scales, uint8_t* qt,
                                     float* scales_t, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (!((block_rows == 1 || block_rows == 128) && block_cols == 128)) return FP8_ERR_SHAPE;
    if (rows < 0 || cols < 0 || rows % 128 != 0 || cols % 128 != 0) return FP8_ERR_SHAPE;
    const int64_t n = checked_count(rows, cols);
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (n == 0) return FP8_OK;
    if (x == nullptr || q == nullptr || scales == nullptr || qt == nullptr || scales_t == nullptr) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(qt, 16) || !aligned(scales, 4) || !aligned(scales_t, 4))
        return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_quant_block_transpose(x, dtype, rows, cols, block_rows, fmt, q, scales, qt, scales_t,
                                                        static_cast<cudaStream_t>(stream)));
}

int fp8_quantize_per_tensor_transpose(const void* x, int dtype, int64_t rows, int64_t cols, int fmt,
                                      const float* scale_in, uint8_t* q, uint8_t* qt, float* scale_out,
                                      float* amax_out, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (rows < 0 || cols < 0) return FP8_ERR_SHAPE;
    const int64_t n = checked_count(rows, cols);
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (scale_out == nullptr) return FP8_ERR_NULL;
    if (scale_in == nullptr && amax_out == nullptr) return FP8_ERR_NULL;
    if (n > 0 && (x == nullptr || qt == nullptr)) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(qt, 16) || !aligned(scale_out, 4) || !aligned(scale_in, 4) ||
        !aligned(amax_out, 4))
        return FP8_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (amax_out != nullptr && fp8q::launch_zero_f32(amax_out, st) != cudaSuccess) return FP8_ERR_CUDA;
    if (n == 0) {
        // no element: the scale of an empty tensor, as fp8_quantize_per_tensor gives it
        return fp8_quantize_per_tensor(x, dtype, 0, fmt, scale_in, q, scale_out, amax_out, stream);
    }
    if (scale_in == nullptr) {
        const cudaError_t e = fp8q::launch_tensor_amax(x, dtype, n, amax_out, st);
        if (e != cudaSuccess) return FP8_ERR_CUDA;
    }
    return status_of(fp8q::launch_tensor_cast_transpose(x, dtype, rows, cols, fmt, scale_in, amax_out, q, qt, scale_out,
                                                        scale_in ? amax_out : nullptr, st));
}

int fp8_amax(const void* x, int dtype, int64_t n, float* amax_out, void* stream) {
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (amax_out == nullptr || (n > 0 && x == nullptr)) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(amax_out, 4)) return FP8_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (fp8q::launch_zero_f32(amax_out, st) != cudaSuccess) return FP8_ERR_CUDA;
    if (n == 0) return FP8_OK;
    return status_of(fp8q::launch_tensor_amax(x, dtype, n, amax_out, st));
}

int fp8_scale_from_amax(const float* amax_in, int fmt, float* scale_out, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (amax_in == nullptr || scale_out == nullptr) return FP8_ERR_NULL;
    if (!aligned(amax_in, 4) || !aligned(scale_out, 4)) return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_scale_from_amax(amax_in, fmt, scale_out, static_cast<cudaStream_t>(stream)));
}

int fp8_quantize_blockwise(const void* x, int dtype, int64_t rows, int64_t cols, int block_rows, int block_cols,
                           int fmt, uint8_t* q, float* scales, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (rows < 0 || cols < 0) return FP8_ERR_SHAPE;
    if (!((block_rows == 1 || block_rows == 128) && block_cols == 128)) return FP8_ERR_SHAPE;
    const int64_t n = checked_count(rows, cols);
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (n == 0) return FP8_OK;  // no element, no block, no scale
    if (x == nullptr || q == nullptr || scales == nullptr) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scales, 4)) return FP8_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (cols % 128 != 0) {
        e = fp8q::launch_quant_block_general(x, dtype, rows, cols, block_rows, block_cols, fmt, q, scales, st);
    } else if (block_rows == 1) {
        e = fp8q::launch_quant_1x128(x, dtype, n / 128, fmt, q, scales, st);
    } else {
        e = fp8q::launch_quant_128x128(x, dtype, rows, cols, fmt, q, scales, st);
    }
    return status_of(e);
}

static_assert(sizeof(fp8_block_tensor) == sizeof(fp8q::GroupTensor) &&
                  offsetof(fp8_block_tensor, x) == offsetof(fp8q::GroupTensor, x) &&
                  offsetof(fp8_block_tensor, q) == offsetof(fp8q::GroupTensor, q) &&
                  offsetof(fp8_block_tensor, scales) == offsetof(fp8q::GroupTensor, scales) &&
                  offsetof(fp8_block_tensor, rows) == offsetof(fp8q::GroupTensor, rows) &&
                  offsetof(fp8_block_tensor, cols) == offsetof(fp8q::GroupTensor, cols),
              "fp8_block_tensor and the launcher's descriptor share one layout");

int fp8_quantize_blockwise_grouped(const fp8_block_tensor* tensors, int count, int dtype, int block_rows,
                                   int block_cols, int fmt, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (count < 0) return FP8_ERR_ARG;
    if (!((block_rows == 1 || block_rows == 128) && block_cols == 128)) return FP8_ERR_SHAPE;
    if (count == 0) return FP8_OK;
    if (tensors == nullptr) return FP8_ERR_NULL;
    for (int i = 0; i < count; ++i) {
        const fp8_block_tensor& t = tensors[i];
        if (t.rows < 0 || t.cols < 0 || t.cols % 128 != 0) return FP8_ERR_SHAPE;
        const int64_t n = checked_count(t.rows, t.cols);
        if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
        if (n == 0) continue;
        if (t.x == nullptr || t.q == nullptr || t.scales == nullptr) return FP8_ERR_NULL;
        if (!aligned(t.x, 16) || !aligned(t.q, 16) || !aligned(t.scales, 4)) return FP8_ERR_ALIGN;
    }
    return status_of(fp8q::launch_quant_grouped(reinterpret_cast<const fp8q::GroupTensor*>(tensors), count, dtype,
                                                block_rows, fmt, static_cast<cudaStream_t>(stream)));
}

int fp8_dequantize(const uint8_t* q, int fmt, int64_t rows, int64_t cols, int block_rows, int block_cols,
                   const float* scales, void* y, int out_dtype, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(out_dtype)) return FP8_ERR_DTYPE;
    if (rows < 0 || cols < 0) return FP8_ERR_SHAPE;
    int mode;
    if (block_rows == 0 && block_cols == 0) mode = 0;
    else if (block_rows == 1 && block_cols == 128) mode = 1;
    else if (block_rows == 128 && block_cols == 128) mode = 2;
    else return FP8_ERR_SHAPE;
    const int64_t n = checked_count(rows, cols);
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (n == 0) return FP8_OK;
    if (q == nullptr || scales == nullptr || y == nullptr) return FP8_ERR_NULL;
    if (!aligned(q, 16) || !aligned(y, 16) || !aligned(scales, 4)) return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_dequant(q, fmt, rows, cols, mode, scales, y, out_dtype,
                                          static_cast<cudaStream_t>(stream)));
}

int fp8_fake_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int block_rows, int block_cols, int fmt,
                      const float* scale_in, void* y, float* scales_out, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (rows < 0 || cols < 0) return FP8_ERR_SHAPE;
    const bool per_tensor = (block_rows == 0 && block_cols == 0);
    if (!per_tensor && !((block_rows == 1 || block_rows == 128) && block_cols == 128)) return FP8_ERR_SHAPE;
    const int64_t n = checked_count(rows, cols);
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (per_tensor && scale_in == nullptr) return FP8_ERR_NULL;
    if (n == 0) return FP8_OK;
    if (x == nullptr || y == nullptr) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(scale_in, 4) || !aligned(scales_out, 4)) return FP8_ERR_ALIGN;
    const size_t esize = dtype == FP8_F32 ? 4 : 2;
    const uintptr_t xb = reinterpret_cast<uintptr_t>(x), yb = reinterpret_cast<uintptr_t>(y);
    const uintptr_t bytes = static_cast<uintptr_t>(n) * esize;
    if (xb != yb && xb < yb + bytes && yb < xb + bytes) return FP8_ERR_ARG;  // partial overlap
    return status_of(fp8q::launch_fake_quant(x, dtype, rows, cols, per_tensor ? 0 : block_rows, fmt, scale_in, y,
                                             per_tensor ? nullptr : scales_out, static_cast<cudaStream_t>(stream)));
}

int fp8_quantize_mx(const void* x, int dtype, int64_t rows, int64_t cols, int fmt, int rule, uint8_t* q,
                    uint8_t* e8m0, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (rule != FP8_MX_FIT && rule != FP8_MX_OCP) return FP8_ERR_ARG;
    if (rows < 0 || cols < 0) return FP8_ERR_SHAPE;
    const int64_t n = checked_count(rows, cols);
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (n == 0) return FP8_OK;
    if (x == nullptr || q == nullptr || e8m0 == nullptr) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16)) return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_quant_mx(x, dtype, rows, cols, fmt, rule, q, e8m0, static_cast<cudaStream_t>(stream)));
}

int fp8_dequantize_mx(const uint8_t* q, int fmt, int64_t rows, int64_t cols, const uint8_t* e8m0, void* y,
                      int out_dtype, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(out_dtype)) return FP8_ERR_DTYPE;
    if (rows < 0 || cols < 0) return FP8_ERR_SHAPE;
    const int64_t n = checked_count(rows, cols);
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (n == 0) return FP8_OK;
    if (q == nullptr || e8m0 == nullptr || y == nullptr) return FP8_ERR_NULL;
    if (!aligned(q, 16) || !aligned(y, 16)) return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_dequant_mx(q, fmt, rows, cols, e8m0, y, out_dtype, static_cast<cudaStream_t>(stream)));
}

int fp8_gemm_blockwise_ex(const uint8_t* a, const float* sa, int a_fmt, const uint8_t* b, const float* sb,
                          int b_block_rows, int b_fmt, int64_t M, int64_t N, int64_t K, void* c, int c_dtype,
                          void* stream) {
    if (!fmt_ok(a_fmt) || !fmt_ok(b_fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(c_dtype)) return FP8_ERR_DTYPE;
    if (b_block_rows != 1 && b_block_rows != 128) return FP8_ERR_SHAPE;
    if (M < 0 || N < 0 || K < 0 || N % 256 != 0 || K % 128 != 0) return FP8_ERR_SHAPE;
    if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF || checked_count(M, N) < 0) return FP8_ERR_SHAPE;
    if (M == 0 || N == 0) return FP8_OK;
    if (c == nullptr) return FP8_ERR_NULL;
    if (!aligned(c, 16)) return FP8_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {  // an empty sum
        const size_t bytes = static_cast<size_t>(M) * static_cast<size_t>(N) * (c_dtype == FP8_F32 ? 4u : 2u);
        return status_of(cudaMemsetAsync(c, 0, bytes, st));
    }
    if (a == nullptr || sa == nullptr || b == nullptr || sb == nullptr) return FP8_ERR_NULL;
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(sa, 4) || !aligned(sb, 4)) return FP8_ERR_ALIGN;
    if (!fp8q::gemm_blockwise_supported()) return FP8_ERR_CUDA;
    return status_of(fp8q::launch_gemm_blockwise(a, sa, a_fmt, b, sb, b_block_rows, b_fmt, M, N, K, c, c_dtype, st));
}

int fp8_gemm_blockwise(const uint8_t* a, const float* sa, int a_fmt, const uint8_t* b, const float* sb, int b_fmt,
                       int64_t M, int64_t N, int64_t K, void* c, int c_dtype, void* stream) {
    return fp8_gemm_blockwise_ex(a, sa, a_fmt, b, sb, 128, b_fmt, M, N, K, c, c_dtype, stream);
}

int fp8_amax_history_update(float* history, int32_t* state, int window, const float* amax, int fmt, float* scale,
                            void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (window <= 0 || window > 65536) return FP8_ERR_ARG;
    if (history == nullptr || state == nullptr || amax == nullptr || scale == nullptr) return FP8_ERR_NULL;
    if (!aligned(history, 4) || !aligned(state, 4) || !aligned(amax, 4) || !aligned(scale, 4)) return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_amax_history_update(history, state, window, amax, fmt, scale,
                                                      static_cast<cudaStream_t>(stream)));
}

int fp8_amax_history_update_ex(float* history, int32_t* state, int window, const float* amax, int fmt, float* scale,
                               int algo, float alpha, float margin, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (window <= 0 || window > 65536) return FP8_ERR_ARG;
    if (algo != FP8_AMAX_WINDOW_MAX && algo != FP8_AMAX_EMA) return FP8_ERR_ARG;
    if (!(alpha >= 0.0f && alpha <= 1.0f) || !(margin > 0.0f)) return FP8_ERR_ARG;
    if (history == nullptr || state == nullptr || amax == nullptr || scale == nullptr) return FP8_ERR_NULL;
    if (!aligned(history, 4) || !aligned(state, 4) || !aligned(amax, 4) || !aligned(scale, 4)) return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_amax_history_update_ex(history, state, window, amax, fmt, scale, algo, alpha, margin,
                                                         static_cast<cudaStream_t>(stream)));
}

int fp8_quantize_delayed_step(const void* x, int dtype, int64_t n, int fmt, float* scale, float* history,
                              int32_t* state, int window, int algo, float alpha, float margin, uint8_t* q,
                              float* scale_used, float* amax_out, void* workspace, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (n < 0 || n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
    if (window <= 0 || window > 65536) return FP8_ERR_ARG;
    if (algo != FP8_AMAX_WINDOW_MAX && algo != FP8_AMAX_EMA) return FP8_ERR_ARG;
    if (!(alpha >= 0.0f && alpha <= 1.0f) || !(margin > 0.0f)) return FP8_ERR_ARG;
    if (scale == nullptr || history == nullptr || state == nullptr || scale_used == nullptr || amax_out == nullptr ||
        workspace == nullptr)
        return FP8_ERR_NULL;
    if (n > 0 && (x == nullptr || q == nullptr)) return FP8_ERR_NULL;
    if (scale_used == scale) return FP8_ERR_ARG;  // the scale is rewritten in place
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale, 4) || !aligned(history, 4) || !aligned(state, 4) ||
        !aligned(scale_used, 4) || !aligned(amax_out, 4) || !aligned(workspace, 16))
        return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_tensor_delayed_step(x, dtype, n, fmt, scale, q, scale_used, amax_out, history,
                                                      state, window, algo, alpha, margin, workspace,
                                                      static_cast<cudaStream_t>(stream)));
}

static_assert(sizeof(fp8_delayed_tensor) == sizeof(fp8q::DelayedTensor) &&
                  offsetof(fp8_delayed_tensor, x) == offsetof(fp8q::DelayedTensor, x) &&
                  offsetof(fp8_delayed_tensor, q) == offsetof(fp8q::DelayedTensor, q) &&
                  offsetof(fp8_delayed_tensor, n) == offsetof(fp8q::DelayedTensor, n) &&
                  offsetof(fp8_delayed_tensor, scale) == offsetof(fp8q::DelayedTensor, scale) &&
                  offsetof(fp8_delayed_tensor, history) == offsetof(fp8q::DelayedTensor, history) &&
                  offsetof(fp8_delayed_tensor, state) == offsetof(fp8q::DelayedTensor, state) &&
                  offsetof(fp8_delayed_tensor, scale_used) == offsetof(fp8q::DelayedTensor, scale_used) &&
                  offsetof(fp8_delayed_tensor, amax_out) == offsetof(fp8q::DelayedTensor, amax_out),
              "fp8_delayed_tensor and the launcher's descriptor share one layout");

int fp8_quantize_delayed_step_grouped(const fp8_delayed_tensor* tensors, int count, int dtype, int fmt, int window,
                                      int algo, float alpha, float margin, void* workspace, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (count < 0) return FP8_ERR_ARG;
    if (window <= 0 || window > 65536) return FP8_ERR_ARG;
    if (algo != FP8_AMAX_WINDOW_MAX && algo != FP8_AMAX_EMA) return FP8_ERR_ARG;
    if (!(alpha >= 0.0f && alpha <= 1.0f) || !(margin > 0.0f)) return FP8_ERR_ARG;
    if (count == 0) return FP8_OK;
    if (tensors == nullptr || workspace == nullptr) return FP8_ERR_NULL;
    if (!aligned(workspace, 16)) return FP8_ERR_ALIGN;
    for (int i = 0; i < count; ++i) {
        const fp8_delayed_tensor& t = tensors[i];
        if (t.n < 0 || t.n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
        if (t.scale == nullptr || t.history == nullptr || t.state == nullptr || t.scale_used == nullptr ||
            t.amax_out == nullptr)
            return FP8_ERR_NULL;
        if (t.n > 0 && (t.x == nullptr || t.q == nullptr)) return FP8_ERR_NULL;
        if (t.scale_used == t.scale) return FP8_ERR_ARG;
        if (!aligned(t.x, 16) || !aligned(t.q, 16) || !aligned(t.scale, 4) || !aligned(t.history, 4) ||
            !aligned(t.state, 4) || !aligned(t.scale_used, 4) || !aligned(t.amax_out, 4))
            return FP8_ERR_ALIGN;
    }
    return status_of(fp8q::launch_tensor_delayed_step_grouped(reinterpret_cast<const fp8q::DelayedTensor*>(tensors),
                                                              count, dtype, fmt, window, algo, alpha, margin,
                                                              workspace, static_cast<cudaStream_t>(stream)));
}

int fp8_quantize_per_tensor_grouped(const fp8_current_tensor* tensors, int count, int dtype, int fmt, void* stream) {
    if (!fmt_ok(fmt)) return FP8_ERR_FORMAT;
    if (!dtype_ok(dtype)) return FP8_ERR_DTYPE;
    if (count < 0) return FP8_ERR_ARG;
    if (count == 0) return FP8_OK;
    if (tensors == nullptr) return FP8_ERR_NULL;
    for (int i = 0; i < count; ++i) {
        const fp8_current_tensor& t = tensors[i];
        if (t.n < 0 || t.n > (INT64_MAX >> 4)) return FP8_ERR_SHAPE;
        if (t.scale_out == nullptr || t.amax_out == nullptr) return FP8_ERR_NULL;
        if (t.n > 0 && (t.x == nullptr || t.q == nullptr)) return FP8_ERR_NULL;
        if (!aligned(t.x, 16) || !aligned(t.q, 16) || !aligned(t.scale_out, 4) || !aligned(t.amax_out, 4))
            return FP8_ERR_ALIGN;
    }
    static_assert(sizeof(fp8_current_tensor) == sizeof(fp8q::CurrentTensor), "descriptor layouts must agree");
    return status_of(fp8q::launch_tensor_current_grouped(reinterpret_cast<const fp8q::CurrentTensor*>(tensors), count,
                                                         dtype, fmt, static_cast<cudaStream_t>(stream)));
}

int fp8_device_status(uint32_t* status, int clear, void* stream) {
    if (status == nullptr) return FP8_ERR_NULL;
    if (!aligned(status, 4)) return FP8_ERR_ALIGN;
    return status_of(fp8q::launch_device_status(status, clear ? 1 : 0, static_cast<cudaStream_t>(stream)));
}

int fp8_selftest_wait_timeout(uint32_t timeout_us, void* stream) {
    if (timeout_us == 0 || timeout_us > 10000000u) return FP8_ERR_ARG;
    return status_of(fp8q::launch_selftest_wait_timeout(static_cast<uint64_t>(timeout_us) * 1000u,
                                                        static_cast<cudaStream_t>(stream)));
}

const char* fp8_status_string(int status) {
    switch (status) {
        case FP8_OK: return "ok";
        case FP8_ERR_NULL: return "a required pointer is NULL";
        case FP8_ERR_SHAPE: return "invalid size or unsupported block shape";
        case FP8_ERR_ALIGN: return "pointer not aligned (tensors: 16 bytes, scalars: 4 bytes)";
        case FP8_ERR_FORMAT: return "fmt is not FP8_E4M3 or FP8_E5M2";
        case FP8_ERR_DTYPE: return "dtype is not FP8_F32 or FP8_BF16";
        case FP8_ERR_CUDA: return "a CUDA call or kernel launch failed";
        case FP8_ERR_ARG: return "invalid argument";
        case FP8_ERR_TOO_LARGE: return "tensor too large for the one-pass kernel of the no-allocation entry point";
        default: return "unknown status";
    }
}

}  // extern "C"
