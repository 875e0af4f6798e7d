/* Exhaustive check, on the CPU, of the division method the quantizer kernels
 * use in place of IEEE binary32 division (the kernels' corrected quotient:
 * Markstein, IBM J. Res. Dev. 34(1), 1990; Muller et al., "Handbook of
 * Floating-Point Arithmetic", division with a fused multiply-add).
 *
 * (1) scale = amax / 448 by q = RN(a y448), s = RN(q + RN(a - 448 q) y448)
 *     with y448 = RN(1/448), for every positive finite BF16 amax: must equal
 *     the IEEE quotient bit for bit.
 * (2) x / s by y = RN(1/s), q = RN(x y), n = RN(q s - x), q' = RN(q - n y), for
 *     every BF16 amax with s >= 2^-92 (smaller scales divide) and every BF16 x
 *     with |x| <= amax, both signs: q' must equal fl32(x / s) bit for bit
 *     wherever |x / s| >= 2^-11 or x = +-0 (signs of zero included), and give
 *     the same saturating round-to-nearest-even E4M3 code everywhere.
 * fmaf is the C library's correctly rounded fused multiply-add; build without
 * floating-point contraction.  Prints one line and exits 0 when every check
 * passes. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t b_of(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

static float e4m3_mag[127];  /* magnitudes of codes 0x00 .. 0x7E */

static void init_e4m3(void) {
    for (int c = 0; c < 127; ++c) {
        const int e = c >> 3, m = c & 7;
        e4m3_mag[c] = e == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
    }
}

/* saturating round-to-nearest-even E4M3 code of a finite float */
static int e4m3_code(float x) {
    float a = fabsf(x);
    if (a > 448.0f) a = 448.0f;
    int lo = 0, hi = 126;
    while (lo < hi) {  /* largest code with magnitude <= a */
        const int mid = (lo + hi + 1) / 2;
        if (e4m3_mag[mid] <= a) lo = mid; else hi = mid - 1;
    }
    int best = lo;
    if (lo < 126) {
        const double d0 = (double)a - e4m3_mag[lo], d1 = (double)e4m3_mag[lo + 1] - a;
        if (d1 < d0 || (d1 == d0 && ((lo + 1) & 1) == 0)) best = lo + 1;
    }
    return (signbit(x) ? 0x80 : 0) | best;
}

int main(void) {
    init_e4m3();
    const float y448 = 0x1.24924ap-9f;
    if (b_of(y448) != b_of(1.0f / 448.0f)) { puts("RN(1/448) constant wrong"); return 1; }
    long n1 = 0, bad1 = 0;
    for (uint32_t a = 1; a <= 0x7F7F; ++a) {
        const float fa = f_of(a << 16);
        const float q = fa * y448;
        const float s = fmaf(fmaf(-q, 448.0f, fa), y448, q);
        ++n1;
        if (b_of(s) != b_of(fa / 448.0f)) ++bad1;
    }
    long n2 = 0, bitdiff = 0, zerobad = 0, codediff = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : n2, bitdiff, zerobad, codediff)
    for (uint32_t a = 1; a <= 0x7F7F; ++a) {
        const float fa = f_of(a << 16);
        const float s = fa / 448.0f;
        if (!(s >= 0x1p-92f)) continue;
        const float y = 1.0f / s;
        for (uint32_t xm = 0; xm <= a; ++xm)
            for (int sg = 0; sg < 2; ++sg) {
                const float x = f_of((xm << 16) | (sg ? 0x80000000u : 0u));
                const float ref = x / s;
                const float q = x * y;
                const float n = fmaf(q, s, -x);
                const float qq = fmaf(-n, y, q);
                ++n2;
                if (b_of(qq) != b_of(ref)) {
                    if (x == 0.0f) ++zerobad;
                    else if (fabsf(ref) >= 0x1p-11f) ++bitdiff;
                    if (e4m3_code(qq) != e4m3_code(ref)) ++codediff;
                }
            }
    }
    printf("scale: %ld amax values, %ld differ; quotient: %ld pairs, %ld bit differences "
           "(|x/s| >= 2^-11), %ld zero-sign errors, %ld code differences\n",
           n1, bad1, n2, bitdiff, zerobad, codediff);
    return (bad1 || bitdiff || zerobad || codediff || n2 < 1000000000L) ? 1 : 0;
}
