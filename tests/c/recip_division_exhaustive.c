/*
 * Exhaustive check of the division scheme used by the dequantize kernels.
 *
 * The kernels compute y = fp32(q / s) without a division per element:
 *     r  = RN(1 / s)               once per scale (a correctly rounded reciprocal)
 *     y0 = RN(q * r)
 *     e  = RN(q - s * y0)          one fused multiply-add
 *     y  = RN(y0 + e * r)          one fused multiply-add
 * Every FP8 value q is (1 + j/8) * 2^a (j = 0..7; E5M2 uses the even j), so as
 * long as no step under- or overflows, scaling q and s by powers of two scales
 * every step exactly, and the scheme is exact for all (q, s) iff it is exact
 * for q in {1, 1.125, ..., 1.875} and every s in [1, 2): 8 * 2^23 cases, all
 * checked here against the correctly rounded quotient.
 *
 * Exit status 0 when every case matches; prints the first mismatches otherwise.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }

int main(void)
{
    long bad = 0, checked = 0;
    for (uint32_t m = 0; m < (1u << 23); ++m) {
        const float s = from_bits(0x3F800000u | m);          /* s in [1, 2) */
        const float r = 1.0f / s;                            /* IEEE: correctly rounded */
        for (int j = 0; j < 8; ++j) {
            const float q = 1.0f + (float)j / 8.0f;
            const float y0 = q * r;
            const float e = fmaf(-y0, s, q);
            const float y = fmaf(e, r, y0);
            const float exact = q / s;                       /* IEEE: correctly rounded */
            ++checked;
            if (y != exact) {
                if (bad < 10) printf("mismatch s=%a q=%a got %a want %a\n", s, q, y, exact);
                ++bad;
            }
        }
    }
    printf("checked %ld cases, %ld mismatches\n", checked, bad);
    return bad != 0;
}
