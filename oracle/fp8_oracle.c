/*
 * fp8_oracle.c -- plain CPU oracle for FP8 scaled quantization.
 *
 * TEST INFRASTRUCTURE, NOT PART OF THE LIBRARY.  Only the test suite, the
 * smoke check and the CPU-baseline leg of the benchmark load this file.  It
 * shares no code, header, table or constant with the CUDA sources, and it
 * includes no CUDA header and uses no library FP8 type: every FP8 code is
 * decoded from, and rounded onto, the value set that the format table defines.
 *
 * It is scalar, single-threaded and slow on purpose, so that a reader can
 * check each step against the pages by eye.
 *
 * Pages (title, address) and the parts followed:
 *   [FP8-native]  "PyTorch native FP8 dtypes: E4M3 / E5M2, delayed scaling,
 *                  conv fallback" (m.nxbn.cn/news/137885)
 *                  s1.2 format table, s1.3 "FN" (finite only, saturating),
 *                  s2.2 scalar experiment, s3.2 FP8QuantizeFunction,
 *                  s4.1 scale = max_val / amax, s4.2 DelayedScaler.
 *   [MP-handbook] "Mixed precision and FP8 training" (anrans.github.io,
 *                  ai-infra-handbooks/train/practice/mixed-precision)
 *                  section "FP8 training": quant / per_tensor / per_block
 *                  code and its printed output; exercise 2.
 *
 * Readings taken where the pages are silent or disagree (each is also listed
 * in the design notes):
 *   R1  E4M3 largest finite value is 448 (format table, MP-handbook output);
 *       code 0x7F/0xFF is therefore not a finite value and decodes to NaN.
 *   R2  Overflow saturates to +-max for both formats ([FP8-native] s1.3,
 *       [MP-handbook] clamp(-MAX, MAX) before the cast); +-Inf in -> +-max.
 *   R3  Rounding is round-to-nearest, ties to the even significand.
 *   R4  The scale multiplies: q = fp8(fp32(x * s)), s = fp32(MAX / amax)
 *       ([FP8-native] s4.1, s4.2 quantize()); dequant divides: y = fp32(q / s).
 *   R5  amax is clamped below by eps = fp32(1e-12) in every mode
 *       ([MP-handbook] per_block clamp(min=1e-12); [FP8-native] s4.2 eps).
 *   R6  Blocks at a ragged edge hold only the elements inside the tensor.
 *   R7  bf16 input is widened to fp32 exactly; bf16 output is the fp32
 *       result rounded once more to bf16, nearest-even.
 *   R14 The delayed-scaling margin divides: s = MAX / (max(amax, eps) * m),
 *       each operation rounded to fp32 ([FP8-native] s4.3).
 *   R15 The moving-average amax: first update m = amax, later ones
 *       m = alpha * amax + (1 - alpha) * m, each product and the sum rounded
 *       to fp32; the scale follows from m once `window` updates are in.
 *   R16 MX blocks: scale 2^k, k by the fit rule or the OCP MX rule (below).
 *   R17 An MX block with an infinite amax gets the NaN scale byte.
 *   R18 The transposed per-tensor output holds the same codes as q.
 *   R19 The consumer GEMM divides each 128-chunk partial sum by the two
 *       block scales (the quantizers' multipliers).
 *   R20 The weight-gradient GEMM takes B with 1x128 blocks along K (the
 *       transposed quantization of an activation): its scale is per row of
 *       B and per chunk, sb[n][c]; otherwise the same sum as R19.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_E4M3 0
#define ORC_E5M2 1
#define ORC_F32 0
#define ORC_BF16 1

#define ORC_OK 0
#define ORC_EBADARG (-1)

/* [FP8-native] s1.2 table: exponent bits, mantissa bits, exponent bias and
 * largest finite value of float8_e4m3fn and float8_e5m2. */
static const int EXP_BITS[2] = {4, 5};
static const int MAN_BITS[2] = {3, 2};
static const int EXP_BIAS[2] = {7, 15};
static const double MAX_FINITE[2] = {448.0, 57344.0};

/* R5: the amax clamp, as an fp32 (the clamp in [MP-handbook] per_block runs
 * on an fp32 tensor). */
static const float AMAX_EPS = 1e-12f;

static int fmt_ok(int fmt) { return fmt == ORC_E4M3 || fmt == ORC_E5M2; }
static int dtype_ok(int dt) { return dt == ORC_F32 || dt == ORC_BF16; }

/* ------------------------------------------------------------------ */
/* Decode: the value of an 8-bit code, from the format table.          */
/* ------------------------------------------------------------------ */

/* [FP8-native] s1.2: sign bit, E exponent bits, M mantissa bits, bias.
 * E == 0 is the subnormal range: m * 2^(1 - bias - M), smallest 2^-9 (E4M3)
 * and 2^-16 (E5M2).  Otherwise (1 + m / 2^M) * 2^(E - bias).  E5M2 keeps the
 * IEEE all-ones exponent for Inf/NaN; E4M3 has no Inf, and its all-ones code
 * 0x7F would be 480 > 448, so it is NaN (reading R1). */
double orc_fp8_decode(int code, int fmt)
{
    if (!fmt_ok(fmt)) return NAN;
    code &= 0xFF;
    const int M = MAN_BITS[fmt];
    const int bias = EXP_BIAS[fmt];
    const int sign = (code >> 7) & 1;
    const int E = (code >> M) & ((1 << EXP_BITS[fmt]) - 1);
    const int m = code & ((1 << M) - 1);
    double mag;
    if (fmt == ORC_E4M3 && (code & 0x7F) == 0x7F) return NAN;
    if (fmt == ORC_E5M2 && E == 31) {
        if (m != 0) return NAN;
        mag = INFINITY;
    } else if (E == 0) {
        mag = ldexp((double)m, 1 - bias - M);
    } else {
        mag = ldexp(1.0 + (double)m / (double)(1 << M), E - bias);
    }
    return sign ? -mag : mag;
}

/* Decoded values of the 128 non-negative codes, cached so the search below
 * does not call ldexp seven times per element.  Filled from orc_fp8_decode. */
static double g_value[2][128];
static int g_top[2];   /* largest non-negative code with a finite value */
static int g_ready = 0;

static void ensure_tables(void)
{
    if (g_ready) return;
    for (int f = 0; f < 2; ++f) {
        for (int c = 0; c < 128; ++c) g_value[f][c] = orc_fp8_decode(c, f);
        int top = 127;
        while (!isfinite(g_value[f][top])) --top;
        g_top[f] = top;
    }
    g_ready = 1;
}

/* 0 when the decoded table agrees with the format table's largest finite
 * value and the non-negative finite codes increase strictly; else -1. */
int orc_selfcheck(void)
{
    ensure_tables();
    for (int f = 0; f < 2; ++f) {
        if (g_value[f][g_top[f]] != MAX_FINITE[f]) return -1;
        for (int c = 1; c <= g_top[f]; ++c)
            if (!(g_value[f][c] > g_value[f][c - 1])) return -1;
    }
    return 0;
}

int orc_fp8_top_code(int fmt)
{
    if (!fmt_ok(fmt)) return -1;
    ensure_tables();
    return g_top[fmt];
}

/* ------------------------------------------------------------------ */
/* Encode: round an fp32 value onto the finite FP8 values.             */
/* ------------------------------------------------------------------ */

/* The definition written out: the nearest finite value of the format (R3:
 * ties go to the code whose last mantissa bit is 0, i.e. the even code,
 * since the non-negative codes 0..top run in value order and the code's low
 * bit is the mantissa's low bit, also across a binade); anything at or above
 * the largest finite value becomes that value (R2).  The sign is carried
 * over, so -0 and negatives that round to zero give 0x80.  NaN stays NaN
 * (0x7F | sign; out of contract). */
int orc_fp8_encode(float v, int fmt)
{
    if (!fmt_ok(fmt)) return -1;
    ensure_tables();
    uint32_t bits;
    memcpy(&bits, &v, sizeof bits);
    const int sign = (bits >> 31) ? 0x80 : 0x00;
    if (isnan(v)) return sign | 0x7F;
    const double a = fabs((double)v);
    const int top = g_top[fmt];
    const double *val = g_value[fmt];
    if (a >= val[top]) return sign | top;
    /* largest code lo with val[lo] <= a; then val[lo] <= a < val[lo + 1] */
    int lo = 0, hi = top;
    while (hi - lo > 1) {
        const int mid = (lo + hi) / 2;
        if (val[mid] <= a) lo = mid; else hi = mid;
    }
    /* both neighbours have at most 4 significant bits, so their midpoint is
     * exact in double, and a (an fp32) compares against it exactly */
    const double midpoint = 0.5 * (val[lo] + val[hi]);
    int c;
    if (a < midpoint) c = lo;
    else if (a > midpoint) c = hi;
    else c = (lo % 2 == 0) ? lo : hi;
    return sign | c;
}

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32                                                       */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an fp32, so widening is exact. */
float orc_bf16_to_f32(uint16_t h)
{
    const uint32_t b = (uint32_t)h << 16;
    float f;
    memcpy(&f, &b, sizeof f);
    return f;
}

/* Nearest bf16, ties to even: keep the upper 16 bits, and round up when the
 * dropped half is above 0x8000, or exactly 0x8000 with an odd kept part.  A
 * carry moves into the exponent, so the binade step and overflow to Inf come
 * out right.  NaN stays a quiet NaN. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t b;
    memcpy(&b, &f, sizeof b);
    if (isnan(f)) return (uint16_t)((b >> 16) | 0x0040);
    uint32_t upper = b >> 16;
    const uint32_t lower = b & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
    return (uint16_t)upper;
}

static float load_elem(const void *x, int dtype, int64_t i)
{
    if (dtype == ORC_F32) return ((const float *)x)[i];
    return orc_bf16_to_f32(((const uint16_t *)x)[i]);
}

/* ------------------------------------------------------------------ */
/* amax, scale, one scaled cast                                        */
/* ------------------------------------------------------------------ */

/* [FP8-native] s4.1: amax is the largest |x|.  NaN is skipped (out of
 * contract).  The empty set gives 0. */
static float amax_of(const void *x, int dtype, int64_t begin, int64_t end)
{
    float m = 0.0f;
    for (int64_t i = begin; i < end; ++i) {
        const float a = fabsf(load_elem(x, dtype, i));
        if (a > m) m = a;
    }
    return m;
}

float orc_amax(const void *x, int dtype, int64_t n)
{
    if (!dtype_ok(dtype) || n < 0) return NAN;
    return amax_of(x, dtype, 0, n);
}

/* [FP8-native] s4.1: scale = max_val / amax, with amax clamped at eps (R5).
 * The quotient is formed in double and rounded once to fp32; for two fp32
 * operands that equals the correctly rounded fp32 quotient (double has more
 * than 2*24+2 bits, so the double rounding is innocuous). */
float orc_scale_from_amax(float amax, int fmt)
{
    if (!fmt_ok(fmt)) return NAN;
    const float m = (amax > AMAX_EPS) ? amax : AMAX_EPS;
    return (float)(MAX_FINITE[fmt] / (double)m);
}

/* [FP8-native] s4.2 quantize(): (x * scale).to(fp8).  The product is an fp32
 * tensor op, so it is rounded to fp32 first (the double product of two fp32
 * numbers is exact, then one rounding), and that fp32 is what gets encoded. */
static uint8_t scaled_code(float x, float s, int fmt)
{
    const float p = (float)((double)x * (double)s);
    return (uint8_t)orc_fp8_encode(p, fmt);
}

/* ------------------------------------------------------------------ */
/* Quantize                                                            */
/* ------------------------------------------------------------------ */

/* Per-tensor scaling ([MP-handbook] per_tensor; [FP8-native] s4.1-s4.2).
 * scale_in == NULL: current scaling, s = scale(amax(x)).
 * scale_in != NULL: delayed scaling, s = *scale_in (a scale made from earlier
 * steps' amax); amax(x) is still reported for the history.
 * Writes q[0..n), *scale_out = s used, *amax_out = amax(x). */
int orc_quantize_per_tensor(const void *x, int dtype, int64_t n, int fmt,
                            const float *scale_in, uint8_t *q,
                            float *scale_out, float *amax_out)
{
    if (!fmt_ok(fmt) || !dtype_ok(dtype) || n < 0) return ORC_EBADARG;
    const float amax = amax_of(x, dtype, 0, n);
    const float s = scale_in ? *scale_in : orc_scale_from_amax(amax, fmt);
    for (int64_t i = 0; i < n; ++i) q[i] = scaled_code(load_elem(x, dtype, i), s, fmt);
    if (scale_out) *scale_out = s;
    if (amax_out) *amax_out = amax;
    return ORC_OK;
}

/* Per-tensor scaling with a transposed second output: qt[c][r] = q[r][c]
 * (x is [rows, cols] row-major, qt is [cols, rows] row-major).  One scale for
 * the whole tensor, so the transposed codes are the same codes in the other
 * order; reading R18: nothing else changes. */
int orc_quantize_per_tensor_transpose(const void *x, int dtype, int64_t rows, int64_t cols, int fmt,
                                      const float *scale_in, uint8_t *q, uint8_t *qt,
                                      float *scale_out, float *amax_out)
{
    if (rows < 0 || cols < 0) return ORC_EBADARG;
    const int rc = orc_quantize_per_tensor(x, dtype, rows * cols, fmt, scale_in, q, scale_out, amax_out);
    if (rc != ORC_OK) return rc;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) qt[c * rows + r] = q[r * cols + c];
    return ORC_OK;
}

/* Fine-grained scaling ([MP-handbook] per_block: one scale per rows x cols
 * block; 1x128 for activations, 128x128 for weights).  x is row-major
 * [rows, cols].  Block (bi, bj) covers rows [bi*br, bi*br+br) and columns
 * [bj*bc, bj*bc+bc), cut at the tensor edge (R6).  scales is row-major
 * [ceil(rows/br), ceil(cols/bc)], one s per block. */
int orc_quantize_blockwise(const void *x, int dtype, int64_t rows, int64_t cols,
                           int br, int bc, int fmt, uint8_t *q, float *scales)
{
    if (!fmt_ok(fmt) || !dtype_ok(dtype) || rows < 0 || cols < 0 || br <= 0 || bc <= 0)
        return ORC_EBADARG;
    const int64_t nbr = (rows + br - 1) / br;
    const int64_t nbc = (cols + bc - 1) / bc;
    for (int64_t bi = 0; bi < nbr; ++bi) {
        const int64_t r0 = bi * br;
        const int64_t r1 = (r0 + br < rows) ? r0 + br : rows;
        for (int64_t bj = 0; bj < nbc; ++bj) {
            const int64_t c0 = bj * bc;
            const int64_t c1 = (c0 + bc < cols) ? c0 + bc : cols;
            float amax = 0.0f;
            for (int64_t r = r0; r < r1; ++r) {
                const float m = amax_of(x, dtype, r * cols + c0, r * cols + c1);
                if (m > amax) amax = m;
            }
            const float s = orc_scale_from_amax(amax, fmt);
            scales[bi * nbc + bj] = s;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c)
                    q[r * cols + c] = scaled_code(load_elem(x, dtype, r * cols + c), s, fmt);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Dequantize                                                          */
/* ------------------------------------------------------------------ */

/* [FP8-native] s4.1 ("divide by the scale to restore") and s4.2
 * (.to(dtype) / scale): y = fp32(decode(q) / s).  br == bc == 0 selects one
 * scale for the whole tensor (scales[0]); otherwise the block layout of
 * orc_quantize_blockwise.  bf16 output rounds that fp32 once more (R7). */
int orc_dequantize(const uint8_t *q, int fmt, int64_t rows, int64_t cols,
                   int br, int bc, const float *scales, void *y, int out_dtype)
{
    if (!fmt_ok(fmt) || !dtype_ok(out_dtype) || rows < 0 || cols < 0) return ORC_EBADARG;
    const int per_tensor = (br == 0 && bc == 0);
    if (!per_tensor && (br <= 0 || bc <= 0)) return ORC_EBADARG;
    const int64_t nbc = per_tensor ? 1 : (cols + bc - 1) / bc;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            const int64_t i = r * cols + c;
            const float s = per_tensor ? scales[0] : scales[(r / br) * nbc + (c / bc)];
            const float v = (float)orc_fp8_decode(q[i], fmt); /* exact: <= 4 significant bits */
            const float out = v / s;                          /* one fp32 division */
            if (out_dtype == ORC_F32) ((float *)y)[i] = out;
            else ((uint16_t *)y)[i] = orc_f32_to_bf16(out);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Delayed scaling: the amax history                                   */
/* ------------------------------------------------------------------ */

/* [FP8-native] s4.3: the scale may keep a margin, max_val / (amax * margin)
 * (the page's example margin is 1.1).  Reading R14: both steps in fp32,
 * s = RN(MAX / RN(max(amax, eps) * margin)); margin 1 gives
 * orc_scale_from_amax exactly. */
static float scale_with_margin(float amax, float margin, int fmt)
{
    const float m = (amax > AMAX_EPS) ? amax : AMAX_EPS;
    const float d = (float)((double)m * (double)margin); /* exact product, one rounding */
    return (float)(MAX_FINITE[fmt] / (double)d);        /* correctly rounded fp32 quotient */
}

/* [FP8-native] s4.2 DelayedScaler.update: append this step's amax to a
 * window of the last `window` amax values; once the window is full, the
 * scale becomes max_val / max(max(window), eps).  Until then it keeps its
 * value (1.0 at the start).  The window is a ring: history[window], with
 * state[0] = next slot, state[1] = number of valid entries. */
int orc_amax_history_update(float *history, int32_t *state, int window,
                            float amax, int fmt, float *scale)
{
    if (!fmt_ok(fmt) || window <= 0) return ORC_EBADARG;
    int32_t pos = state[0], count = state[1];
    if (pos < 0 || pos >= window || count < 0 || count > window) return ORC_EBADARG;
    history[pos] = amax;
    pos = (pos + 1) % window;
    if (count < window) count += 1;
    if (count == window) {
        float m = 0.0f;
        for (int i = 0; i < window; ++i)
            if (history[i] > m) m = history[i];
        *scale = orc_scale_from_amax(m, fmt);
    }
    state[0] = pos;
    state[1] = count;
    return ORC_OK;
}

/* Delayed scaling with the [FP8-native] s4.3 refinements.
 *   algo 0 (window max): as orc_amax_history_update, but the refreshed scale
 *          keeps the margin: MAX / (max(max(window), eps) * margin).
 *   algo 1 (EMA): the amax is smoothed instead of windowed (s4.2 names an
 *          exponential moving average as Transformer Engine's smoothing).
 *          history[0] holds the average m: the first update sets m = amax,
 *          later ones m = RN(RN(alpha*amax) + RN(RN(1 - alpha) * m)) in fp32
 *          (reading R15).  state[1] counts updates (saturating at window);
 *          once it reaches window the scale becomes MAX / (max(m, eps) *
 *          margin) at every update -- window acts as the warm-up length.
 *          state[0] is unused. */
int orc_amax_history_update_ex(float *history, int32_t *state, int window, float amax, int fmt,
                               float *scale, int algo, float alpha, float margin)
{
    if (!fmt_ok(fmt) || window <= 0 || (algo != 0 && algo != 1)) return ORC_EBADARG;
    if (!(margin > 0.0f) || !(alpha >= 0.0f && alpha <= 1.0f)) return ORC_EBADARG;
    int32_t pos = state[0], count = state[1];
    if (count < 0 || count > window) return ORC_EBADARG;
    if (algo == 0) {
        if (pos < 0 || pos >= window) return ORC_EBADARG;
        history[pos] = amax;
        pos = (pos + 1) % window;
        if (count < window) count += 1;
        if (count == window) {
            float m = 0.0f;
            for (int i = 0; i < window; ++i)
                if (history[i] > m) m = history[i];
            *scale = scale_with_margin(m, margin, fmt);
        }
    } else {
        if (count == 0) {
            history[0] = amax;
        } else {
            const float beta = (float)(1.0 - (double)alpha);
            const float a_part = (float)((double)alpha * (double)amax);
            const float m_part = (float)((double)beta * (double)history[0]);
            history[0] = (float)((double)a_part + (double)m_part);
        }
        if (count < window) count += 1;
        if (count == window) *scale = scale_with_margin(history[0], margin, fmt);
    }
    state[0] = pos;
    state[1] = count;
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* MX blocks: 1x32 with a power-of-two scale                           */
/* ------------------------------------------------------------------ */

/* [MP-handbook] "FP8 training", last notes: Blackwell's MX formats (MXFP8)
 * let every 32 consecutive elements share one scale factor, in hardware.  That
 * scale is a power of two, s = 2^k, stored as the E8M0 byte of the dequant
 * multiplier 2^-k (byte = 127 - k; E8M0 is an unsigned exponent with bias 127
 * whose byte 0xFF means NaN).
 * Reading R16: which k --
 *   rule 0 (fit): the largest k with max(amax, eps) * 2^k <= MAX, i.e. the
 *                 pages' s = MAX / amax restricted to a power of two; no
 *                 element of the block saturates.
 *   rule 1 (OCP MX): k = emax_elem - floor(log2(max(amax, eps))), emax_elem
 *                 the exponent of the format's largest normal (8 for E4M3, 15
 *                 for E5M2); the top of a binade can saturate.
 * Reading R17: a block holding +-Inf has an infinite amax and no power of two
 * that fits; it gets k = 0 for its elements and the NaN byte 0xFF, so its
 * dequantized values are all NaN.  (NaN elements are skipped by amax, as in
 * every other mode.)
 * Elements: q = fp8(fp32(x * 2^k)), as in every other mode. */
static int mx_exponent(float amax, int fmt, int rule)
{
    if (isinf(amax)) return 0;
    const double a = (double)((amax > AMAX_EPS) ? amax : AMAX_EPS);
    const int emax_elem = (fmt == ORC_E4M3) ? 8 : 15;
    int e; /* frexp: a = f * 2^e with f in [0.5, 1), so floor(log2 a) = e - 1 */
    (void)frexp(a, &e);
    int k = emax_elem - (e - 1);
    if (rule == 1) return k;
    /* fit: the OCP exponent is at most one too large; step down until
     * a * 2^k <= MAX holds (exact in double) */
    while (ldexp(a, k) > MAX_FINITE[fmt]) --k;
    return k;
}

static uint8_t mx_byte(float amax, int k)
{
    return isinf(amax) ? (uint8_t)0xFF : (uint8_t)(127 - k);
}

int orc_mx_exponent(float amax, int fmt, int rule)
{
    if (!fmt_ok(fmt) || (rule != 0 && rule != 1)) return -1000;
    return mx_exponent(amax, fmt, rule);
}

/* x [rows, cols]; blocks of 32 consecutive elements of a row (the last one in
 * a row may be short); e8m0 [rows, ceil(cols / 32)]. */
int orc_quantize_mx(const void *x, int dtype, int64_t rows, int64_t cols, int fmt, int rule,
                    uint8_t *q, uint8_t *e8m0)
{
    if (!fmt_ok(fmt) || !dtype_ok(dtype) || rows < 0 || cols < 0 || (rule != 0 && rule != 1))
        return ORC_EBADARG;
    const int64_t nbc = (cols + 31) / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t bj = 0; bj < nbc; ++bj) {
            const int64_t c0 = bj * 32, c1 = (c0 + 32 < cols) ? c0 + 32 : cols;
            const float amax = amax_of(x, dtype, r * cols + c0, r * cols + c1);
            const int k = mx_exponent(amax, fmt, rule);
            const float s = (float)ldexp(1.0, k);
            e8m0[r * nbc + bj] = mx_byte(amax, k);
            for (int64_t c = c0; c < c1; ++c)
                q[r * cols + c] = scaled_code(load_elem(x, dtype, r * cols + c), s, fmt);
        }
    }
    return ORC_OK;
}

/* MX dequant: y = fp32(decode(q) * 2^(byte - 127)), the MX value being the
 * element times the shared scale; for a byte made by the quantizer that is
 * the real number decode(q) / 2^k.  Byte 0xFF (NaN) gives NaN. */
int orc_dequantize_mx(const uint8_t *q, int fmt, int64_t rows, int64_t cols, const uint8_t *e8m0,
                      void *y, int out_dtype)
{
    if (!fmt_ok(fmt) || !dtype_ok(out_dtype) || rows < 0 || cols < 0) return ORC_EBADARG;
    const int64_t nbc = (cols + 31) / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            const int64_t i = r * cols + c;
            const uint8_t b = e8m0[r * nbc + c / 32];
            const double xs = (b == 0xFF) ? NAN : ldexp(1.0, (int)b - 127);
            const float out = (float)(orc_fp8_decode(q[i], fmt) * xs);
            if (out_dtype == ORC_F32) ((float *)y)[i] = out;
            else ((uint16_t *)y)[i] = orc_f32_to_bf16(out);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Consumer: blockwise-scaled FP8 GEMM                                 */
/* ------------------------------------------------------------------ */

/* [MP-handbook] "FP8 training", closing notes: FP8 inputs with fp32
 * accumulation; the tensor-core partial sum is promoted every 128 elements,
 * where the 1x128 (activation) and 128x128 (weight) scales are applied.
 * Reading R19: with the quantizers' multiplier scales,
 *   C[m][n] = sum over chunks c of (sum_{k in c} decode(a[m][k]) *
 *             decode(b[n][k])) / (sa[m][c] * sb[n/128][c]).
 * a [M, K], b [N, K] row-major codes; sa [M, ceil(K/128)],
 * sb [ceil(N/128), ceil(K/128)]; c [M, N] in double.  Each product of two
 * FP8 values is exact in double, the chunk sums and the quotient are rounded
 * in double only: the result is the real value to within a few double ulps.
 * b_block_rows 1 (reading R20): B holds 1x128 blocks, sb [N, ceil(K/128)],
 * and the divisor is sa[m][c] * sb[n][c]. */
int orc_gemm_blockwise_ex(const uint8_t *a, const float *sa, int a_fmt, const uint8_t *b, const float *sb,
                          int b_block_rows, int b_fmt, int64_t M, int64_t N, int64_t K, double *c)
{
    if (!fmt_ok(a_fmt) || !fmt_ok(b_fmt) || M < 0 || N < 0 || K < 0) return ORC_EBADARG;
    if (b_block_rows != 1 && b_block_rows != 128) return ORC_EBADARG;
    const int64_t nkc = (K + 127) / 128;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t kc = 0; kc < nkc; ++kc) {
                const int64_t k0 = kc * 128, k1 = (k0 + 128 < K) ? k0 + 128 : K;
                double p = 0.0;
                for (int64_t k = k0; k < k1; ++k)
                    p += orc_fp8_decode(a[m * K + k], a_fmt) * orc_fp8_decode(b[n * K + k], b_fmt);
                acc += p / ((double)sa[m * nkc + kc] * (double)sb[(n / b_block_rows) * nkc + kc]);
            }
            c[m * N + n] = acc;
        }
    }
    return ORC_OK;
}

int orc_gemm_blockwise(const uint8_t *a, const float *sa, int a_fmt, const uint8_t *b, const float *sb,
                       int b_fmt, int64_t M, int64_t N, int64_t K, double *c)
{
    return orc_gemm_blockwise_ex(a, sa, a_fmt, b, sb, 128, b_fmt, M, N, K, c);
}
