// fp8q_launch.h -- internal host-side launchers of libfp8q (not part of the ABI).
//
// The C ABI (fp8q_abi.cu) validates arguments and calls these; each one picks
// a launch shape for the current device and enqueues kernels on `stream`.
// They return the first CUDA error seen (cudaSuccess when all launches went
// in).  None of them allocates or synchronizes.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp8q {

// Number of SMs of the current device (cached per device).
int device_sm_count();

// 1x128 blocks over a [rows, cols] tensor with cols % 128 == 0: the blocks
// are the n / 128 consecutive 128-element runs, scales are one per run.
cudaError_t launch_quant_1x128(const void* x, int dtype, int64_t nblocks, int fmt,
                               uint8_t* q, float* scales, cudaStream_t stream);

// Grouped blockwise quantization: `count` tensors (cols % 128 == 0 each) in
// as few launches as possible (up to 128 tensors per launch).
struct GroupTensor {
    const void* x;
    uint8_t* q;
    float* scales;
    int64_t rows;
    int64_t cols;
};
cudaError_t launch_quant_grouped(const GroupTensor* tensors, int count, int dtype, int block_rows, int fmt,
                                 cudaStream_t stream);

// 128x128 blocks over [rows, cols], cols % 128 == 0, any rows.
cudaError_t launch_quant_128x128(const void* x, int dtype, int64_t rows, int64_t cols, int fmt,
                                 uint8_t* q, float* scales, cudaStream_t stream);

// MX: 1x32 blocks with power-of-two scales stored as E8M0 bytes
// [rows, ceil(cols / 32)]; rule 0 = fit, 1 = OCP MX.
cudaError_t launch_quant_mx(const void* x, int dtype, int64_t rows, int64_t cols, int fmt, int rule, uint8_t* q,
                            uint8_t* e8m0, cudaStream_t stream);
cudaError_t launch_dequant_mx(const uint8_t* q, int fmt, int64_t rows, int64_t cols, const uint8_t* e8m0, void* y,
                              int out_dtype, cudaStream_t stream);

// Delayed scaling with a margin and a choice of window max (algo 0) or EMA (algo 1).
cudaError_t launch_amax_history_update_ex(float* history, int32_t* state, int window, const float* amax, int fmt,
                                          float* scale, int algo, float alpha, float margin, cudaStream_t stream);

// FP8 GEMM with blockwise scales on the tcgen05 tensor cores:
// C[M, N] = sum over 128-wide K chunks of (A_c B_c^T) / (sa * sb), A [M, K]
// codes with 1x128 scales sa [M, K/128], B [N, K] codes with 128x128 scales
// sb [N/128, K/128] (b_block_rows 128) or 1x128 scales sb [N, K/128]
// (b_block_rows 1).  Needs N % 256 == 0, K % 128 == 0, K > 0.
bool gemm_blockwise_supported();
cudaError_t launch_gemm_blockwise(const uint8_t* a, const float* sa, int a_fmt, const uint8_t* b, const float* sb,
                                  int b_block_rows, int b_fmt, int64_t M, int64_t N, int64_t K, void* c,
                                  int c_dtype, cudaStream_t stream);

// Device address of the status word of the current device (nullptr on failure).
unsigned int* device_status_word();

// One-pass per-tensor current scaling (cooperative launch, 16-byte workspace).
// Sets *launched = false (and enqueues nothing) when x is too large for one
// pass; the caller then takes the two-pass path.
cudaError_t launch_tensor_fused(const void* x, int dtype, int64_t n, int fmt, uint8_t* q, float* scale_out,
                                float* amax_out, void* workspace, cudaStream_t stream, bool* launched);

// Whether x (n elements) is small enough for the one-pass kernel: 1 yes, 0 no,
// -1 unknown (a CUDA query failed, or the device has no cooperative launch).
int tensor_fused_fit(const void* x, int dtype, int64_t n, int fmt);

// The one-pass kernel with its workspace in a fixed array of this module's
// device memory instead of caller memory (see quant_tensor_fused.cu).  The
// caller has checked tensor_fused_fit first.
cudaError_t launch_tensor_fused_noalloc(const void* x, int dtype, int64_t n, int fmt, uint8_t* q, float* scale_out,
                                        float* amax_out, cudaStream_t stream);

// Copy the device status word to out[0] (device memory), clearing it if asked.
cudaError_t launch_device_status(unsigned int* out, int clear, cudaStream_t stream);

// A single-thread kernel whose bounded wait can only time out (sets the
// wait-timeout status bit after limit_ns).
cudaError_t launch_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

// Any block shape, any cols (ragged right edge), element-wise accesses.
cudaError_t launch_quant_block_general(const void* x, int dtype, int64_t rows, int64_t cols,
                                       int block_rows, int block_cols, int fmt,
                                       uint8_t* q, float* scales, cudaStream_t stream);

// Per-tensor: amax of x into *amax_out (which the caller has zeroed).
cudaError_t launch_tensor_amax(const void* x, int dtype, int64_t n, float* amax_out,
                               cudaStream_t stream);

// *scale_out = MAX / max(*amax_in, eps) (one thread).
cudaError_t launch_scale_from_amax(const float* amax_in, int fmt, float* scale_out, cudaStream_t stream);
// *p = 0, in stream order (one thread).
cudaError_t launch_zero_f32(float* p, cudaStream_t stream);

// Per-tensor cast.  scale_in == nullptr: s from *amax_in (current scaling);
// else s = *scale_in (delayed), and amax_out (if non-null, zeroed by the
// caller) receives amax(x) from the same pass.  *scale_out = s.
cudaError_t launch_tensor_cast(const void* x, int dtype, int64_t n, int fmt,
                               const float* scale_in, const float* amax_in,
                               uint8_t* q, float* scale_out, float* amax_out,
                               cudaStream_t stream);

// Per-tensor cast with a transposed second output qt [cols, rows] (q [rows,
// cols] optional).  Scale arguments as in launch_tensor_cast.
// Blockwise quantization of x and of x^T in one pass (rows, cols multiples of
// 128; block_rows 1 for 1x128, 128 for 128x128).
cudaError_t launch_quant_block_transpose(const void* x, int dtype, int64_t rows, int64_t cols, int block_rows,
                                         int fmt, uint8_t* q, float* scales, uint8_t* qt, float* scales_t,
                                         cudaStream_t stream);
cudaError_t launch_tensor_cast_transpose(const void* x, int dtype, int64_t rows, int64_t cols, int fmt,
                                         const float* scale_in, const float* amax_in, uint8_t* q, uint8_t* qt,
                                         float* scale_out, float* amax_out, cudaStream_t stream);

// One delayed-scaling step in one launch: cast with *scale, amax(x), then (in
// the last CTA) the history update that rewrites *scale.  16-byte workspace,
// zero before the first call and left zero.
cudaError_t launch_tensor_delayed_step(const void* x, int dtype, int64_t n, int fmt, float* scale, uint8_t* q,
                                       float* scale_used, float* amax_out, float* history, int32_t* state,
                                       int window, int algo, float alpha, float margin, void* workspace,
                                       cudaStream_t stream);

// The same for `count` tensors in as few launches as possible (up to 96 per
// launch); workspace: one 16-byte slot per tensor, zero before the first call.
struct DelayedTensor {
    const void* x;
    uint8_t* q;
    int64_t n;
    float* scale;
    float* history;
    int32_t* state;
    float* scale_used;
    float* amax_out;
};
cudaError_t launch_tensor_delayed_step_grouped(const DelayedTensor* tensors, int count, int dtype, int fmt, int window,
                                               int algo, float alpha, float margin, void* workspace,
                                               cudaStream_t stream);

// Per-tensor current scaling of many tensors: zero every amax_out, one amax
// pass and one cast pass over all of them (up to 128 tensors per launch).
struct CurrentTensor {
    const void* x;
    uint8_t* q;
    int64_t n;
    float* scale_out;
    float* amax_out;
};
cudaError_t launch_tensor_current_grouped(const CurrentTensor* tensors, int count, int dtype, int fmt,
                                          cudaStream_t stream);

// Fused quantize -> dequantize round trip in x's dtype.  block_rows 0: per
// tensor with *scale_in; 1 or 128: block scales (written to `scales` if it is
// non-null).
cudaError_t launch_fake_quant(const void* x, int dtype, int64_t rows, int64_t cols, int block_rows, int fmt,
                              const float* scale_in, void* y, float* scales, cudaStream_t stream);

// Dequantize.  mode 0: per-tensor; 1: 1x128; 2: 128x128.
cudaError_t launch_dequant(const uint8_t* q, int fmt, int64_t rows, int64_t cols, int mode,
                           const float* scales, void* y, int out_dtype, cudaStream_t stream);

// Delayed-scaling history update (one warp).
cudaError_t launch_amax_history_update(float* history, int32_t* state, int window,
                                       const float* amax, int fmt, float* scale,
                                       cudaStream_t stream);

}  // namespace fp8q
