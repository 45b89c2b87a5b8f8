/*
 * fp8q.h -- C ABI of libfp8q, FP8 scaled quantization on NVIDIA B200 (sm_100a).
 *
 * The library computes the data-parallel path of FP8 mixed-precision
 * training described on two pages:
 *   [FP8-native]  PyTorch native FP8 dtypes (m.nxbn.cn/news/137885):
 *                 s1.2 format table, s1.3 finite-only saturation,
 *                 s4.1 scale = max_val / amax, s4.2 delayed scaling.
 *   [MP-handbook] Mixed precision and FP8 training (anrans.github.io,
 *                 ai-infra-handbooks/train/practice/mixed-precision),
 *                 section "FP8 training": per-tensor vs 1x128 / 128x128
 *                 block scaling (quant, per_tensor, per_block).
 *
 * Arithmetic of the quantizers:
 *   amax  = max |x| over the scaled group (a block, or the whole tensor)
 *   s     = fp32( MAX / max(amax, 1e-12f) ),  MAX = 448 (E4M3), 57344 (E5M2)
 *           (per tensor, per 1x128 or 128x128 block; MX blocks of 1x32 use
 *           a power of two instead, see fp8_quantize_mx)
 *   q     = fp8_rne_satfinite( fp32(x * s) )   x widened to fp32 exactly
 *   y     = fp32( decode(q) / s ),  bf16 output = bf16_rne(y)
 * The stored scale is the multiplier s (not its reciprocal).  Casts round to
 * nearest-even and saturate: no Inf is ever produced, and E4M3 has no Inf.
 * fp8_gemm_blockwise consumes 1x128 and 128x128 codes on the tensor cores.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or keeps them (the no-allocation entry
 *     point uses a fixed array of the library's own device memory).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream), never synchronizes, and is
 *     safe to call from several host threads.  Calls that touch the same
 *     buffers must be ordered by the caller (same stream or events).
 *   - Tensors are contiguous and row-major, [rows, cols] with cols innermost.
 *   - x, q and y must be 16-byte aligned; scale, amax and history pointers
 *     4-byte aligned.  Anything else returns FP8_ERR_ALIGN.
 *   - Arguments are checked before anything is launched; on an error return
 *     nothing has been enqueued.  A launch failure returns FP8_ERR_CUDA.
 *     Faults inside a kernel surface at the caller's next synchronization,
 *     as with any CUDA work.
 *   - Element counts may be 0 (nothing is launched unless a scale or amax
 *     output has to be written).
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* FP8 formats ([FP8-native] s1.2): E4M3 = float8_e4m3fn (bias 7, max 448,
 * no Inf, 0x7F/0xFF are NaN); E5M2 = float8_e5m2 (bias 15, max 57344). */
enum fp8_format { FP8_E4M3 = 0, FP8_E5M2 = 1 };

/* Element types of high-precision tensors. */
enum fp8_dtype { FP8_F32 = 0, FP8_BF16 = 1 };

/* Status codes.  0 is success; every error is negative. */
enum fp8_status {
    FP8_OK = 0,
    FP8_ERR_NULL = -1,          /* a required pointer is NULL */
    FP8_ERR_SHAPE = -2,         /* negative size, or an unsupported block shape */
    FP8_ERR_ALIGN = -3,         /* a pointer is not aligned as stated above */
    FP8_ERR_FORMAT = -4,        /* fmt is not an fp8_format */
    FP8_ERR_DTYPE = -5,         /* dtype is not an fp8_dtype */
    FP8_ERR_CUDA = -6,          /* a CUDA call or launch failed */
    FP8_ERR_ARG = -7,           /* any other invalid argument (e.g. window <= 0) */
    FP8_ERR_TOO_LARGE = -8      /* larger than fp8_quantize_per_tensor_fused_noalloc can take */
};

/*
 * Per-tensor quantization: one scale for the whole tensor.
 * Follows [MP-handbook] "FP8 training" per_tensor and [FP8-native] s4.1-s4.2.
 *
 *   x          [n] input, dtype FP8_F32 or FP8_BF16 (any n >= 0)
 *   scale_in   NULL: current scaling -- s is computed from amax(x) in this
 *              call (two passes over x: amax, then cast).
 *              non-NULL: delayed scaling -- device pointer to one fp32 scale
 *              made from earlier steps (e.g. by fp8_amax_history_update);
 *              x is cast with it in one pass, values beyond range saturate.
 *   q          [n] output codes (uint8 bit patterns of fmt)
 *   scale_out  [1] output: the scale used.  May equal scale_in.
 *   amax_out   [1] output: amax(x) (0 for n == 0).  Required with current
 *              scaling; with delayed scaling it may be NULL, which skips the
 *              amax reduction.
 * Errors: FP8_ERR_NULL (x or q NULL with n > 0, scale_out NULL, amax_out
 * NULL with scale_in NULL), FP8_ERR_SHAPE (n < 0), FP8_ERR_ALIGN,
 * FP8_ERR_FORMAT, FP8_ERR_DTYPE, FP8_ERR_CUDA.
 */
int fp8_quantize_per_tensor(const void *x, int dtype, int64_t n, int fmt,
                            const float *scale_in, uint8_t *q,
                            float *scale_out, float *amax_out, void *stream);

/*
 * Per-tensor CURRENT scaling in one pass over x, for tensors small enough to
 * be held on chip by the CTAs that fit on the GPU at once (on a B200 up to
 * 18.5 MiB of input when x is 32-byte aligned, 11.6 MiB when it is only
 * 16-byte aligned: the exact element counts are stated with
 * fp8_quantize_per_tensor_fused_noalloc).  Larger tensors transparently take
 * the two-pass path of fp8_quantize_per_tensor and do not touch the
 * workspace.  Same results as fp8_quantize_per_tensor with scale_in == NULL.
 *
 *   x, dtype, n, fmt, q, scale_out, amax_out   as fp8_quantize_per_tensor
 *              (scale_out and amax_out both required)
 *   workspace  FP8_FUSED_WORKSPACE_BYTES of caller-owned device memory,
 *              16-byte aligned, zeroed once before its first use; every call
 *              leaves it ready for the next one (it keeps a count of
 *              completed calls and the last amax), and zeroing it again
 *              between calls is also allowed.  Calls that share a workspace
 *              must not overlap on the device (use one workspace per stream).
 *              After FP8_DEVICE_STATUS_WAIT_TIMEOUT, zero it before reuse.
 * The one-pass kernel holds its slice of x in registers, meets the other CTAs
 * at a grid-wide barrier (a cooperative launch, so every CTA is resident),
 * and then casts.  The barrier wait gives up after about a second, sets
 * FP8_DEVICE_STATUS_WAIT_TIMEOUT and leaves the codes unwritten.
 * Errors: those of fp8_quantize_per_tensor; FP8_ERR_NULL or FP8_ERR_ALIGN
 * for the workspace.
 */
#define FP8_FUSED_WORKSPACE_BYTES 16
int fp8_quantize_per_tensor_fused(const void *x, int dtype, int64_t n, int fmt,
                                  uint8_t *q, float *scale_out, float *amax_out,
                                  void *workspace, void *stream);

/*
 * fp8_quantize_per_tensor_fused without a workspace argument, for callers that
 * cannot allocate device memory: code that runs where cudaMalloc is not
 * allowed or not safe (it synchronizes the device and can fail under memory
 * pressure), such as a plugin called by an inference runtime that offers no
 * workspace, or a C caller whose device memory is all owned by another
 * framework's allocator.  (The pages have no counterpart: this is an
 * interface convenience, not part of the method.)
 *
 * Same arguments and results as fp8_quantize_per_tensor_fused minus the
 * workspace.  Instead, the workspace lives in a fixed 256-byte array in the
 * library's own device memory (16 bytes of it are used), which every GPU that
 * loads the library keeps until the process exits.  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - The first call on each device looks up that array's device address
 *     (cudaGetSymbolAddress) with the device current; make that first call
 *     before any stream capture.  The address is cached per device for the
 *     life of the process, so do not call this entry point after
 *     cudaDeviceReset (the library's device memory may then have moved).
 *   - Every call clears the workspace (cudaMemsetAsync) before its launch.
 *   - All calls share the one array: calls that can overlap on the GPU
 *     (different streams without ordering between them) race and give wrong
 *     results.  Order such calls, or use fp8_quantize_per_tensor_fused with
 *     one workspace per stream.
 *   - Limit: only tensors that fit the one-pass kernel are accepted; larger
 *     ones return FP8_ERR_TOO_LARGE with nothing enqueued.  The kernel holds
 *     x in the registers of the CTAs (256 threads, 4 lane vectors each) that
 *     can be resident at once, so the largest n is
 *         C * 1024 * E + (E - 1)
 *     with E the elements per lane vector and C the co-resident CTAs:
 *       x 32-byte aligned: 32-byte lanes, E = 16 (bf16) or 8 (fp32);
 *       x only 16-byte aligned: 16-byte lanes, E = 8 (bf16) or 4 (fp32);
 *       C = CTAs per SM (from the kernel's registers) x SMs.
 *     On a B200 (148 SMs) as built here: C = 592 for 32-byte lanes (4 per
 *     SM) and 740 for 16-byte lanes (5 per SM), so n <= 9,699,343 bf16 or
 *     4,849,671 fp32 at a 32-byte-aligned x (18.5 MiB), and n <= 6,062,087
 *     bf16 or 3,031,043 fp32 at an x that is only 16-byte aligned
 *     (11.6 MiB).  The same tensor can therefore be accepted at one address
 *     and refused at another.
 *     n == 0 writes amax 0 and its scale, as the other per-tensor calls do.
 * Errors: those of fp8_quantize_per_tensor_fused (without the workspace
 * ones); FP8_ERR_TOO_LARGE; FP8_ERR_CUDA also when the capacity cannot be
 * known (a failed CUDA query, or a device without cooperative launch).
 */
int fp8_quantize_per_tensor_fused_noalloc(const void *x, int dtype, int64_t n, int fmt,
                                          uint8_t *q, float *scale_out, float *amax_out,
                                          void *stream);

/*
 * amax of a tensor: *amax_out = max |x| (0 for n == 0).  [FP8-native] s4.1.
 * The first step of per-tensor current scaling, exposed on its own so that a
 * tensor sharded over several GPUs can all-reduce (MAX) the shards' amax
 * before the scale is formed.
 *   x          [n], FP8_F32 or FP8_BF16
 *   amax_out   [1] fp32 output (device)
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN, FP8_ERR_DTYPE,
 * FP8_ERR_CUDA.
 */
int fp8_amax(const void *x, int dtype, int64_t n, float *amax_out, void *stream);

/*
 * The scale from an amax: *scale_out = fp32(MAX / max(*amax_in, 1e-12f)).
 * [FP8-native] s4.1.  Both pointers are device pointers (one fp32 each) and
 * may be equal.
 * Errors: FP8_ERR_NULL, FP8_ERR_ALIGN, FP8_ERR_FORMAT, FP8_ERR_CUDA.
 */
int fp8_scale_from_amax(const float *amax_in, int fmt, float *scale_out, void *stream);

/*
 * Fine-grained (blockwise) quantization: one scale per block_rows x
 * block_cols block, in one fused pass (amax, scale, cast, scale store).
 * Follows [MP-handbook] "FP8 training" per_block: 1x128 blocks for
 * activations, 128x128 blocks for weights.
 *
 *   x          [rows, cols] input, FP8_F32 or FP8_BF16
 *   block_rows, block_cols   (1, 128) or (128, 128); anything else is
 *              FP8_ERR_SHAPE
 *   q          [rows, cols] output codes
 *   scales     [ceil(rows / block_rows), ceil(cols / 128)] fp32, row-major;
 *              scales[i][j] is the s of the block whose top-left element is
 *              (i * block_rows, j * 128).
 * Ragged edges: when rows or cols is not a multiple of the block, the last
 * blocks hold only the elements inside the tensor (their amax is taken over
 * those elements).  cols % 128 == 0 takes the fast kernels; other widths
 * take a slower general kernel with the same results.
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN, FP8_ERR_FORMAT,
 * FP8_ERR_DTYPE, FP8_ERR_CUDA.
 */
int fp8_quantize_blockwise(const void *x, int dtype, int64_t rows, int64_t cols,
                           int block_rows, int block_cols, int fmt,
                           uint8_t *q, float *scales, void *stream);

/*
 * Grouped blockwise quantization: fp8_quantize_blockwise over `count`
 * tensors, with the same codes and scales as one call per tensor, in as few
 * launches as possible (up to 128 tensors share one).  For the many small
 * weights and activations of a training step, whose single launches are
 * dominated by their fixed cost.
 *
 *   tensors    host array of `count` descriptors (read during the call; the
 *              pointers in them are device pointers, as in
 *              fp8_quantize_blockwise)
 *   block_rows, block_cols   (1, 128) or (128, 128), for all tensors
 * Every tensor needs cols % 128 == 0 (FP8_ERR_SHAPE otherwise; ragged
 * widths go through fp8_quantize_blockwise).  Empty tensors are skipped.
 * Errors: those of fp8_quantize_blockwise; FP8_ERR_ARG for count < 0.
 */
typedef struct fp8_block_tensor {
    const void *x;      /* [rows, cols] input, dtype */
    uint8_t *q;         /* [rows, cols] codes */
    float *scales;      /* block scales, the layout of fp8_quantize_blockwise */
    int64_t rows;
    int64_t cols;
} fp8_block_tensor;
int fp8_quantize_blockwise_grouped(const fp8_block_tensor *tensors, int count, int dtype,
                                   int block_rows, int block_cols, int fmt, void *stream);

/*
 * Dequantization: y = fp32(decode(q) / s), with s the scale of q's block.
 * Follows [FP8-native] s4.1 (divide by the scale to restore) and s4.2
 * quantize() (.to(dtype) / scale).
 *
 *   q          [rows, cols] codes of fmt
 *   block_rows, block_cols   (0, 0): per-tensor, scales[0] for everything;
 *              (1, 128) or (128, 128): the scale layout of
 *              fp8_quantize_blockwise.
 *   scales     fp32 scales (multipliers, as produced by the quantizers)
 *   y          [rows, cols] output, out_dtype FP8_F32 or FP8_BF16 (bf16 is
 *              the fp32 quotient rounded to nearest-even)
 * Results are bit-exact IEEE quotients for every scale.  NaN codes give NaN.
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN, FP8_ERR_FORMAT,
 * FP8_ERR_DTYPE, FP8_ERR_CUDA.
 */
int fp8_dequantize(const uint8_t *q, int fmt, int64_t rows, int64_t cols,
                   int block_rows, int block_cols, const float *scales,
                   void *y, int out_dtype, void *stream);

/*
 * Fake quantization: the quantize -> dequantize round trip in one pass,
 *   y = RN_dtype( RN_f32( decode(q) / s ) ),  q = fp8( RN_f32(x * s) ),
 * in x's own dtype.  No codes are written.  Follows [FP8-native] s3.2
 * (FP8QuantizeFunction forward: scale, cast to FP8, cast back) and s4.2
 * DelayedScaler.quantize(), and [MP-handbook] "FP8 training" quant().
 *
 *   x, y       [rows, cols] of dtype (FP8_F32 or FP8_BF16); y may be x
 *              (in place) but must not otherwise overlap it
 *   block_rows, block_cols   (1, 128) or (128, 128): s from each block's
 *              amax, as in fp8_quantize_blockwise (ragged edges allowed);
 *              (0, 0): one scale for the tensor, given by scale_in
 *   scale_in   (0, 0) only: device pointer to the fp32 scale (required)
 *   scales_out block modes only: where to write the block scales (layout of
 *              fp8_quantize_blockwise), or NULL to not write them
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN, FP8_ERR_FORMAT,
 * FP8_ERR_DTYPE, FP8_ERR_CUDA.
 */
int fp8_fake_quantize(const void *x, int dtype, int64_t rows, int64_t cols,
                      int block_rows, int block_cols, int fmt,
                      const float *scale_in, void *y, float *scales_out,
                      void *stream);

/*
 * Per-tensor quantization with a second, transposed copy of the codes:
 * qt[c][r] = q[r][c], for a consumer that reads the tensor along its other
 * dimension (the weight-gradient GEMM reads activations and output gradients
 * transposed).  Scaling exactly as fp8_quantize_per_tensor ([MP-handbook]
 * per_tensor; [FP8-native] s4.1-4.2, current or delayed): with one scale for
 * the whole tensor the transposed codes are the same codes, moved.
 *
 *   x          [rows, cols] input, FP8_F32 or FP8_BF16
 *   scale_in   NULL: current scaling (amax pass, then the cast); else the
 *              delayed scale (device fp32), one pass
 *   q          [rows, cols] codes, or NULL to write only qt
 *   qt         [cols, rows] codes (required)
 *   scale_out, amax_out   as in fp8_quantize_per_tensor
 * Tiles of 128x128 go through shared memory; rows % 16 == 0 and
 * cols % 16 == 0 take the vectorised path for full tiles, everything else an
 * element-wise path with the same results.
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN (x, q, qt: 16 bytes),
 * FP8_ERR_FORMAT, FP8_ERR_DTYPE, FP8_ERR_CUDA.
 */
int fp8_quantize_per_tensor_transpose(const void *x, int dtype, int64_t rows, int64_t cols,
                                      int fmt, const float *scale_in, uint8_t *q,
                                      uint8_t *qt, float *scale_out, float *amax_out,
                                      void *stream);

/*
 * Blockwise quantization of x together with that of its transpose, from one
 * read of x.  Follows [MP-handbook] "FP8 training", per_block (1x128
 * activation blocks, 128x128 weight blocks, s = MAX / max(amax, 1e-12f) per
 * block): the weight- and data-gradient GEMMs read their operands along the
 * other dimension, so they need x^T quantized by the same rule.
 *
 *   x          [rows, cols] row-major input, FP8_F32 or FP8_BF16; rows and
 *              cols multiples of 128
 *   block      (1, 128) or (128, 128)
 *   q, scales  exactly fp8_quantize_blockwise(x, block): codes [rows, cols],
 *              scales [rows, cols/128] (1x128) or [rows/128, cols/128]
 *   qt, scales_t
 *              exactly fp8_quantize_blockwise(x^T, block): codes [cols, rows]
 *              and scales [cols, rows/128] (1x128: one scale per 128
 *              elements of a column of x) or [cols/128, rows/128] (128x128:
 *              the same blocks as x, so qt = q^T and scales_t = scales^T)
 * All four outputs are required.  Bit-exact with the two separate calls.
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE (other blocks; rows or cols not a
 * multiple of 128), FP8_ERR_ALIGN (x, q, qt: 16 bytes; scales: 4),
 * FP8_ERR_FORMAT, FP8_ERR_DTYPE, FP8_ERR_CUDA.
 */
int fp8_quantize_blockwise_transpose(const void *x, int dtype, int64_t rows, int64_t cols,
                                     int block_rows, int block_cols, int fmt, uint8_t *q,
                                     float *scales, uint8_t *qt, float *scales_t, void *stream);

/*
 * MX quantization: blocks of 32 consecutive elements of a row share one
 * power-of-two scale.  Follows [MP-handbook] "FP8 training", closing notes
 * (Blackwell's MX formats, MXFP8: every 32 elements share a scale factor in
 * hardware).  For each block, s = 2^k and q = fp8(RN_f32(x * s)); the scale
 * is stored as the E8M0 byte 127 - k, i.e. the exponent of the dequant
 * multiplier 2^-k (the MX shared-scale encoding, bias 127, 0xFF = NaN).
 *
 *   x          [rows, cols] input, FP8_F32 or FP8_BF16
 *   rule       FP8_MX_FIT: the largest k with max(amax, 1e-12f) * 2^k <= MAX
 *              (the pages' MAX / amax rounded down to a power of two; no
 *              element saturates).  FP8_MX_OCP: k = emax - floor(log2(
 *              max(amax, 1e-12f))) with emax 8 (E4M3) or 15 (E5M2), the OCP
 *              MX rule; elements in the top of a binade may saturate.
 *   q          [rows, cols] output codes
 *   e8m0       [rows, ceil(cols / 32)] uint8, row-major (no alignment rule)
 * A block holding +-Inf gets the byte 0xFF and k = 0 for its elements.  NaN
 * elements do not count toward amax.  Ragged right edge: the last block of
 * a row holds cols % 32 elements.  cols % 32 == 0 takes the vectorised
 * kernel; other widths a slower kernel with the same results.
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN (x, q: 16 bytes),
 * FP8_ERR_FORMAT, FP8_ERR_DTYPE, FP8_ERR_ARG (unknown rule), FP8_ERR_CUDA.
 */
enum fp8_mx_rule { FP8_MX_FIT = 0, FP8_MX_OCP = 1 };
int fp8_quantize_mx(const void *x, int dtype, int64_t rows, int64_t cols,
                    int fmt, int rule, uint8_t *q, uint8_t *e8m0, void *stream);

/*
 * MX dequantization: y = RN_f32(decode(q) * 2^(e8m0 - 127)) with the byte of
 * q's block (the layout of fp8_quantize_mx); byte 0xFF gives NaN.  For bytes
 * made by fp8_quantize_mx this is the real quotient decode(q) / s, so it is
 * exact except where it leaves the fp32 range.  bf16 output is that fp32
 * rounded to nearest-even.
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN (q, y: 16 bytes),
 * FP8_ERR_FORMAT, FP8_ERR_DTYPE, FP8_ERR_CUDA.
 */
int fp8_dequantize_mx(const uint8_t *q, int fmt, int64_t rows, int64_t cols,
                      const uint8_t *e8m0, void *y, int out_dtype, void *stream);

/*
 * The consumer of the blockwise codes: an FP8 GEMM on the tensor cores with
 * the fine-grained scales applied in fp32 every 128 products.  Follows
 * [MP-handbook] "FP8 training", closing notes (FP8 inputs, fp32 accumulation;
 * the FP8 accumulator is promoted to CUDA cores every 128 elements, where the
 * 1x128 / 128x128 scales are applied):
 *     C[m][n] = sum over K chunks c of 128:
 *               (sum_{k in c} decode(a[m][k]) * decode(b[n][k])) / (sa[m][c] * sb[n/128][c])
 *
 *   a, a_fmt   [M, K] codes, row-major (K contiguous): an activation
 *              quantized with 1x128 blocks (fp8_quantize_blockwise)
 *   sa         [M, K/128] fp32 scales of a (the quantizer's multipliers)
 *   b, b_fmt   [N, K] codes, row-major: a weight stored [out, in], quantized
 *              with 128x128 blocks
 *   sb         [N/128, K/128] fp32 scales of b
 *   c, c_dtype [M, N] output, FP8_F32 or FP8_BF16 (the fp32 sum rounded to
 *              nearest-even)
 * The per-chunk products run on tcgen05 tensor cores (kind::f8f6f4, fp32
 * accumulator in tensor memory); each chunk's partial sum is multiplied by
 * RN(1 / RN(sa * sb)) and added in fp32 (fma).  Results agree with the exact
 * sum within the accumulation error of that arithmetic (not bit-exact: the
 * tensor cores' summation order is theirs).
 * Shapes: N % 256 == 0 and K % 128 == 0 (else FP8_ERR_SHAPE); any M.  K == 0
 * writes zeros.  M, N, K < 2^31.
 * Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN (a, b, c: 16 bytes;
 * sa, sb: 4), FP8_ERR_FORMAT, FP8_ERR_DTYPE, FP8_ERR_CUDA (also when the
 * driver offers no tensor-map encoder).
 */
int fp8_gemm_blockwise(const uint8_t *a, const float *sa, int a_fmt,
                       const uint8_t *b, const float *sb, int b_fmt,
                       int64_t M, int64_t N, int64_t K,
                       void *c, int c_dtype, void *stream);

/*
 * fp8_gemm_blockwise with a choice of B's scale blocks.  b_block_rows 128 is
 * fp8_gemm_blockwise.  b_block_rows 1 takes B [N, K] quantized with 1x128
 * blocks along K, sb [N, K/128]: the weight-gradient product dW = dY^T X,
 * where both operands are activations (or their gradients) quantized along
 * the token dimension (fp8_quantize_blockwise_transpose gives them):
 *     C[m][n] = sum over K chunks c of 128:
 *               (sum_{k in c} decode(a[m][k]) * decode(b[n][k])) / (sa[m][c] * sb[n][c])
 * With 1x128 B each chunk's partial sum is multiplied by RN(1 / sa) and by
 * RN(1 / sb[n]) and added in fp32; the bound on the error is that of
 * fp8_gemm_blockwise.  Other arguments, shapes and errors as there, plus
 * FP8_ERR_SHAPE for b_block_rows other than 1 or 128.
 */
int fp8_gemm_blockwise_ex(const uint8_t *a, const float *sa, int a_fmt,
                          const uint8_t *b, const float *sb, int b_block_rows, int b_fmt,
                          int64_t M, int64_t N, int64_t K,
                          void *c, int c_dtype, void *stream);

/*
 * Delayed scaling: push one amax into the amax history and refresh the scale.
 * Follows [FP8-native] s4.2 DelayedScaler.update: the last `window` amax
 * values are kept; once `window` of them have been seen, the scale becomes
 * MAX / max(max(history), 1e-12f); before that it is left unchanged.
 *
 *   history    [window] fp32 ring buffer (device)
 *   state      [2] int32 (device): state[0] = next slot, state[1] = number
 *              of valid entries (saturates at window)
 *   amax       [1] fp32 (device): this step's amax, e.g. the amax_out of
 *              fp8_quantize_per_tensor
 *   scale      [1] fp32 (device), in/out
 * Before the first step the caller zeroes history and state and sets
 * *scale = 1.0f.  The state is plain device memory: copying history, state
 * and scale checkpoints and restores it.  A state outside its range is
 * clamped into range on the device (pos taken modulo window, count clamped
 * to [0, window]) rather than faulting.
 * One single-warp launch; runs entirely on the device, no host sync.
 * Errors: FP8_ERR_NULL, FP8_ERR_ALIGN, FP8_ERR_FORMAT, FP8_ERR_ARG
 * (window <= 0 or window > 65536), FP8_ERR_CUDA.
 */
int fp8_amax_history_update(float *history, int32_t *state, int window,
                            const float *amax, int fmt, float *scale,
                            void *stream);

/*
 * Delayed scaling with the refinements of [FP8-native] s4.3 (keep a margin,
 * smooth the amax) -- the same state and call pattern as
 * fp8_amax_history_update.
 *
 *   algo       FP8_AMAX_WINDOW_MAX: the window of fp8_amax_history_update;
 *              once full, scale = MAX / RN(max(max(window), eps) * margin).
 *              FP8_AMAX_EMA: history[0] holds a moving average m of amax
 *              (s4.2 names this smoothing): the first update sets m = amax,
 *              later ones m = RN(RN(alpha*amax) + RN(RN(1-alpha) * m)), all
 *              in fp32.  state[1] counts updates up to `window` (a warm-up);
 *              from then on every update sets
 *              scale = MAX / RN(max(m, eps) * margin).  state[0] is unused and
 *              history needs only 1 element (window is still the warm-up).
 *   alpha      EMA weight of the new amax, in [0, 1] (ignored by WINDOW_MAX)
 *   margin     > 0; 1.0 keeps the plain scale (the page's example is 1.1)
 * With algo = FP8_AMAX_WINDOW_MAX and margin = 1 the results equal
 * fp8_amax_history_update's.  Initialise history and state to zero and
 * *scale to 1.0f as there.
 * Errors: those of fp8_amax_history_update; FP8_ERR_ARG for an unknown
 * algo, alpha outside [0, 1] or margin <= 0 (NaN included).
 */
enum fp8_amax_algo { FP8_AMAX_WINDOW_MAX = 0, FP8_AMAX_EMA = 1 };
int fp8_amax_history_update_ex(float *history, int32_t *state, int window,
                               const float *amax, int fmt, float *scale,
                               int algo, float alpha, float margin, void *stream);

/*
 * One delayed-scaling step in one launch: exactly fp8_quantize_per_tensor with
 * scale_in = scale (the delayed scale of [FP8-native] s4.2) followed by
 * fp8_amax_history_update_ex (s4.2-4.3) on this step's amax, which rewrites
 * *scale for the next step.  The CTA that finishes last performs the
 * update, so no second launch and no host round trip is needed.
 *
 *   x, dtype, n, fmt, q   as in fp8_quantize_per_tensor
 *   scale      [1] fp32 (device), in: this step's scale; out: the next one
 *   history, state, window, algo, alpha, margin   as in
 *              fp8_amax_history_update_ex
 *   scale_used [1] fp32 (device): the scale this step used (must not be
 *              `scale`)
 *   amax_out   [1] fp32 (device): amax(x)
 *   workspace  FP8_FUSED_WORKSPACE_BYTES of device memory, zero before the
 *              first call and left zero by every call; calls that share it
 *              must not overlap on the device
 * Errors: those of the two calls it replaces; FP8_ERR_ARG also when
 * scale_used == scale.
 */
int fp8_quantize_delayed_step(const void *x, int dtype, int64_t n, int fmt,
                              float *scale, float *history, int32_t *state, int window,
                              int algo, float alpha, float margin,
                              uint8_t *q, float *scale_used, float *amax_out,
                              void *workspace, void *stream);

/*
 * fp8_quantize_delayed_step for `count` tensors, in as few launches as
 * possible (up to 128 tensors share one): every tensor's codes, scale, amax,
 * history and state come out exactly as from its own call.  All tensors share
 * dtype, fmt, window, algo, alpha and margin.  For the many small activations
 * and gradients of a training step, whose single launches are dominated by
 * their fixed cost.
 *
 *   tensors    host array of `count` descriptors (read during the call);
 *              each holds the device pointers of one
 *              fp8_quantize_delayed_step call and its element count n
 *   workspace  count * FP8_FUSED_WORKSPACE_BYTES of device memory, zero
 *              before the first call and left zero; slot i belongs to
 *              tensors[i]
 * Errors: those of fp8_quantize_delayed_step, for any tensor; FP8_ERR_ARG
 * also for count < 0.
 */
typedef struct fp8_delayed_tensor {
    const void *x;      /* [n] input */
    uint8_t *q;         /* [n] codes */
    int64_t n;
    float *scale;       /* [1] in: this step's scale; out: the next one */
    float *history;     /* [window] */
    int32_t *state;     /* [2] */
    float *scale_used;  /* [1] */
    float *amax_out;    /* [1] */
} fp8_delayed_tensor;
int fp8_quantize_delayed_step_grouped(const fp8_delayed_tensor *tensors, int count, int dtype,
                                      int fmt, int window, int algo, float alpha, float margin,
                                      void *workspace, void *stream);

/*
 * Per-tensor current scaling (fp8_quantize_per_tensor with scale_in NULL) of
 * `count` tensors in three launches per 128 tensors, whatever their sizes:
 * every amax_out is cleared, then one amax pass and one cast pass run over the
 * chunks of all the tensors.  Each tensor gets its own amax and scale: its
 * codes, scale_out and amax_out come out exactly as from its own call.  All
 * tensors share dtype and fmt.  [MP-handbook] "FP8 training" per_tensor;
 * [FP8-native] s4.1.  For the many small tensors of a training step, whose
 * single calls are dominated by their fixed cost.
 *
 *   tensors    host array of `count` descriptors (read during the call);
 *              each holds the device pointers of one current-scaling
 *              fp8_quantize_per_tensor call and its element count n.  The
 *              scale_out and amax_out words of different tensors must be
 *              distinct (each amax is cleared, then reduced into atomically).
 * Errors: those of fp8_quantize_per_tensor with current scaling, for any
 * tensor; FP8_ERR_ARG for count < 0.
 */
typedef struct fp8_current_tensor {
    const void *x;      /* [n] input */
    uint8_t *q;         /* [n] codes */
    int64_t n;
    float *scale_out;   /* [1] the scale used */
    float *amax_out;    /* [1] amax(x) */
} fp8_current_tensor;
int fp8_quantize_per_tensor_grouped(const fp8_current_tensor *tensors, int count, int dtype, int fmt,
                                    void *stream);

/* Static, human-readable text for a status code (never NULL). */
const char *fp8_status_string(int status);

/* ---- Diagnostics (no counterpart on the pages) ---------------------------
 * Kernels that wait (the grid-wide barrier of the one-pass per-tensor kernel,
 * the mbarrier waits of the GEMM) never wait forever: each wait gives up after
 * about a second, the kernel returns, and it records the event in a device
 * status word.  Results of that launch are then incomplete.
 *
 * The status word is the library's one piece of mutable state besides the
 * no-allocation entry point's scratch array: one word per device, shared by
 * every stream, thread and caller on it.  It is written only when a wait
 * gives up, which does not happen in normal operation.  A set bit says that
 * some launch on this device timed out since the word was last cleared, not
 * which one; a caller that needs to know which call it was clears the word,
 * orders that call alone, and reads the word after it.  The word's address
 * is cached per device, so the library must not be used after
 * cudaDeviceReset.
 *
 * Device status bits: */
#define FP8_DEVICE_STATUS_WAIT_TIMEOUT 0x1u

/*
 * Enqueue a copy of the device status word of the current device into
 * *status (a DEVICE pointer to one uint32), resetting the word to 0 when
 * `clear` is nonzero.  Read *status after synchronizing the stream.
 * Errors: FP8_ERR_NULL, FP8_ERR_ALIGN (status not 4-byte aligned),
 * FP8_ERR_CUDA.
 */
int fp8_device_status(uint32_t *status, int clear, void *stream);

/*
 * Self-test of the bounded wait: launch one thread that runs the same wait as
 * the one-pass kernel's barrier on a word that nothing changes; after
 * timeout_us microseconds it gives up and sets
 * FP8_DEVICE_STATUS_WAIT_TIMEOUT.  The device stays usable.
 * Errors: FP8_ERR_ARG (timeout_us == 0 or > 10 s), FP8_ERR_CUDA.
 */
int fp8_selftest_wait_timeout(uint32_t timeout_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
