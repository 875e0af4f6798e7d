/*
 * oracle.c -- plain, slow CPU oracle for the W8A8 FP8 block-scaled linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant with the
 * CUDA library; every value it needs is derived here from the format
 * definitions.
 *
 * What it computes (page "ProCreations/Nanbeige4.3-33B-FP8", introduction and
 * section "Recipe and calibration"): W8A8 FP8 quantization with E4M3 weights
 * in 128x128 blocks (standard min-max, data independent) and dynamic
 * per-token / group-128 activation scales; the linear layer then multiplies
 * the quantized operands and emits BF16.
 *
 * The library specification fixes the details the page leaves open:
 *   scale = amax / 448 as one IEEE binary32 division (round to nearest even),
 *   an all-zero group gets scale 1.0,
 *   code  = E4M3 value nearest to fl32(x / scale), ties to the even mantissa,
 *           magnitudes above 448 saturate to 448 (never the NaN code),
 *   the GEMM reference is the FP64 sum over k of the dequantized operands
 *   (code * scale) -- the order the GPU promotes in is not part of the result's
 *   definition, only of its rounding.
 *
 * Build: gcc -O2 -fopenmp -fno-fast-math -ffp-contract=off -shared -fPIC.
 * x86-64 evaluates float expressions in binary32 (FLT_EVAL_METHOD 0) and keeps
 * subnormals unless fast-math flags are given, so every float operation below
 * is the IEEE operation it reads as.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GROUP 128 /* channels per activation group; rows and cols of a weight block */

/* BF16 is the upper half of a binary32 pattern, so widening is exact. */
static float bf16_bits_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * E4M3 "fn" format (OCP 8-bit floating point, the variant the page names
 * "e4m3fn"): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities, and S.1111.111 reserved for NaN.  Normal values are
 * (1 + m/8) * 2^(e-7) for e = 1..15 (e = 15 only for m <= 6, so the largest is
 * 1.75 * 2^8 = 448); subnormals are (m/8) * 2^-6.
 */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ((double)m / 8.0) * ldexp(1.0, -6);
    else
        v = (1.0 + (double)m / 8.0) * ldexp(1.0, e - 7);
    return sign ? -v : v;
}

/* Round a non-negative real (held exactly in a double) to the nearest integer,
 * ties to the even integer. */
static double round_half_even(double n)
{
    double lo = floor(n);
    double frac = n - lo; /* exact: n has at most 53 significant bits */
    if (frac > 0.5)
        return lo + 1.0;
    if (frac < 0.5)
        return lo;
    return (fmod(lo, 2.0) == 0.0) ? lo : lo + 1.0;
}

/* Bit pattern of a non-negative value that is exactly an E4M3 value <= 448. */
static uint8_t e4m3_bits_of_exact(double v)
{
    int E;
    if (v == 0.0)
        return 0;
    (void)frexp(v, &E);   /* v = f * 2^E, f in [0.5, 1) */
    int e = E - 1;        /* floor(log2 v) */
    if (e < -6) {         /* subnormal: v = m * 2^-9 */
        int m = (int)(v / ldexp(1.0, -9));
        return (uint8_t)m;
    }
    int m = (int)(v / ldexp(1.0, e - 3)) - 8; /* v = (8 + m) * 2^(e-3) */
    return (uint8_t)(((e + 7) << 3) | m);
}

/*
 * Encode a finite binary32 value: round to the nearest point of the E4M3 grid
 * (ties to even mantissa), then saturate magnitudes above 448 to 448.
 * Within the binade [2^e, 2^(e+1)) the grid spacing is 2^(e-3); below 2^-6
 * (the subnormal range) it stays 2^-9.  The sign is kept, so -0 gives 0x80.
 */
uint8_t oracle_e4m3_encode(float y)
{
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a == 0.0)
        return sign;
    int E;
    (void)frexp(a, &E);
    int e = E - 1;
    if (e < -6)
        e = -6;
    double quantum = ldexp(1.0, e - 3);
    double n = a / quantum;                 /* exact: division by a power of two */
    double v = round_half_even(n) * quantum; /* may round up into the next binade */
    if (v > 448.0)
        v = 448.0;
    return sign | e4m3_bits_of_exact(v);
}

void oracle_e4m3_encode_array(const float *y, int64_t n, uint8_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_e4m3_encode(y[i]);
}

void oracle_e4m3_decode_array(const uint8_t *c, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_e4m3_decode(c[i]);
}

/* scale of a group or block from its amax: amax / 448 in binary32, or 1 for zero */
static float scale_from_amax(float amax)
{
    if (amax == 0.0f)
        return 1.0f;
    return amax / 448.0f;
}

/*
 * Dynamic per-token, group-128 activation quantization.
 * x: BF16 bit patterns [M, K] row-major; q: E4M3 codes [M, K]; s: FP32 [M, K/128].
 * Group g of row m is channels [128 g, 128 g + 128) of that row.
 */
void oracle_quantize_act(const uint16_t *x, int64_t M, int64_t K, uint8_t *q, float *s)
{
    int64_t G = K / GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t g = 0; g < G; g++) {
            const uint16_t *xg = x + m * K + g * GROUP;
            float amax = 0.0f;
            for (int i = 0; i < GROUP; i++) {
                float a = fabsf(bf16_bits_to_float(xg[i]));
                if (a > amax)
                    amax = a;
            }
            float sc = scale_from_amax(amax);
            s[m * G + g] = sc;
            for (int i = 0; i < GROUP; i++) {
                float y = bf16_bits_to_float(xg[i]) / sc;
                q[m * K + g * GROUP + i] = oracle_e4m3_encode(y);
            }
        }
    }
}

/*
 * Same as oracle_quantize_act, restricted to the listed rows.  Output row r of
 * q / s holds input row rows[r].
 */
void oracle_quantize_act_rows(const uint16_t *x, int64_t M, int64_t K, const int64_t *rows,
                              int64_t nrows, uint8_t *q, float *s)
{
    int64_t G = K / GROUP;
    (void)M;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; r++)
        oracle_quantize_act(x + rows[r] * K, 1, K, q + r * K, s + r * G);
}

/*
 * Offline 128x128 block min-max weight quantization.
 * w: BF16 bit patterns [N, K] (out x in, row-major); q: E4M3 [N, K];
 * s: FP32 [N/128, K/128].  Block (i, j) is rows [128 i, +128) x cols [128 j, +128).
 */
void oracle_quantize_weight(const uint16_t *w, int64_t N, int64_t K, uint8_t *q, float *s)
{
    int64_t NB = N / GROUP, KB = K / GROUP;
#pragma omp parallel for schedule(static) collapse(2)
    for (int64_t bi = 0; bi < NB; bi++) {
        for (int64_t bj = 0; bj < KB; bj++) {
            float amax = 0.0f;
            for (int r = 0; r < GROUP; r++)
                for (int c = 0; c < GROUP; c++) {
                    float a = fabsf(bf16_bits_to_float(w[(bi * GROUP + r) * K + bj * GROUP + c]));
                    if (a > amax)
                        amax = a;
                }
            float sc = scale_from_amax(amax);
            s[bi * KB + bj] = sc;
            for (int r = 0; r < GROUP; r++)
                for (int c = 0; c < GROUP; c++) {
                    int64_t idx = (bi * GROUP + r) * K + bj * GROUP + c;
                    q[idx] = oracle_e4m3_encode(bf16_bits_to_float(w[idx]) / sc);
                }
        }
    }
}

/*
 * FP64 reference of the block-scaled GEMM, Y = A * W^T with
 *   A[m, k] = decode(qa[m, k]) * sa[m, k/128]
 *   W[n, k] = decode(qw[n, k]) * sw[n/128, k/128]
 * and out[r, n] = sum over k = 0..K-1 (ascending) of A[rows[r], k] * W[n, k],
 * accumulated in double.  Only the listed rows of A are evaluated, so large
 * shapes can be checked on a sample; pass rows = 0..M-1 for all of them.
 * qa / sa are indexed by the original row number.
 */
void oracle_gemm_ref(const uint8_t *qa, const float *sa, const uint8_t *qw, const float *sw,
                     int64_t M, int64_t N, int64_t K, const int64_t *rows, int64_t nrows,
                     double *out)
{
    int64_t KB = K / GROUP;
    const int64_t NCHUNK = 128;
    (void)M;
    double *arows = (double *)malloc(sizeof(double) * (size_t)(nrows * K));
    double *wrows = (double *)malloc(sizeof(double) * (size_t)(NCHUNK * K));
    if (!arows || !wrows) {
        free(arows);
        free(wrows);
        for (int64_t i = 0; i < nrows * N; i++)
            out[i] = NAN;
        return;
    }
    /* dequantize the requested activation rows once */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; r++) {
        int64_t m = rows[r];
        for (int64_t k = 0; k < K; k++)
            arows[r * K + k] = oracle_e4m3_decode(qa[m * K + k]) * (double)sa[m * KB + k / GROUP];
    }
    for (int64_t n0 = 0; n0 < N; n0 += NCHUNK) {
        int64_t nc = (N - n0 < NCHUNK) ? (N - n0) : NCHUNK;
        /* dequantize a chunk of weight rows */
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < nc; j++) {
            int64_t n = n0 + j;
            for (int64_t k = 0; k < K; k++)
                wrows[j * K + k] =
                    oracle_e4m3_decode(qw[n * K + k]) * (double)sw[(n / GROUP) * KB + k / GROUP];
        }
        /* plain dot products */
#pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < nrows; r++) {
            const double *a = arows + r * K;
            for (int64_t j = 0; j < nc; j++) {
                const double *w = wrows + j * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; k++)
                    acc += a[k] * w[k];
                out[r * N + n0 + j] = acc;
            }
        }
    }
    free(arows);
    free(wrows);
}

/* BF16 rounding of a double, nearest-even on the BF16 grid (8 significant bits),
 * through binary32 first only when that is exact; used to express the
 * closed-form expectations of the exact-arithmetic tests. */
uint16_t oracle_bf16_round(double v)
{
    /* Decompose v exactly and round its significand to 8 bits, ties to even. */
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    int E;
    (void)frexp(a, &E);
    int e = E - 1;                 /* floor(log2 a) */
    if (e < -126)
        e = -126;                  /* BF16 subnormals share the smallest normal quantum */
    double quantum = ldexp(1.0, e - 7);
    double r = round_half_even(a / quantum) * quantum;
    if (r >= ldexp(1.0, 128))
        return sign | 0x7F80;      /* overflow to infinity */
    float f = (float)r;            /* exact: r has <= 8 significant bits in range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

/*
 * FP8 E4M3 KV-cache write with unit scales (page "ProCreations/Nanbeige4.3-33B-FP8",
 * section "Serving" and the "Speed on Vega" table: --kv-cache-dtype fp8_e4m3
 * with unit cache scales).  Each K and V element x is stored as the code of
 * fl32(x / 1) = x under the same rule as every other code here: nearest E4M3,
 * ties to even, saturating at 448.  The page defines no behaviour for
 * non-finite projections; this oracle gives NaN the NaN code (0x7F, sign kept)
 * and +-infinity the saturated code +-448.
 *
 * k, v      : BF16 bit patterns, row t at k + t * row_stride (elements); width
 *             elements per row (all KV heads of the token)
 * loc       : int64 [T], the cache slot of each row
 * k_cache,
 * v_cache   : E4M3 codes, slot s at k_cache + s * slot_stride (bytes)
 * Rows whose slot is outside [0, num_slots) are not written; the count of such
 * rows is returned.
 */
static uint8_t kv_code(uint16_t h)
{
    float x = bf16_bits_to_float(h);
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x))
        return sign | 0x7F;
    if (isinf(x))
        return sign | 0x7E;
    return oracle_e4m3_encode(x / 1.0f);
}

int64_t oracle_kv_write(const uint16_t *k, const uint16_t *v, int64_t row_stride, int64_t T,
                        int64_t width, const int64_t *loc, int64_t num_slots,
                        int64_t slot_stride, uint8_t *k_cache, uint8_t *v_cache)
{
    int64_t skipped = 0;
    for (int64_t t = 0; t < T; t++) {
        int64_t s = loc[t];
        if (s < 0 || s >= num_slots) {
            skipped++;
            continue;
        }
        for (int64_t i = 0; i < width; i++) {
            k_cache[s * slot_stride + i] = kv_code(k[t * row_stride + i]);
            v_cache[s * slot_stride + i] = kv_code(v[t * row_stride + i]);
        }
    }
    return skipped;
}

/*
 * SiLU-gated product feeding the down projection (page "ProCreations/
 * Nanbeige4.3-33B-FP8", introduction: every linear layer, the MLP's down
 * projection included, takes dynamically quantized activations).  The fused
 * gate/up output gu is [M, 2I]: gate = columns [0, I), up = [I, 2I).
 *   h[m, i] = silu(gate) * up = gate / (1 + exp(-gate)) * up, here in FP64.
 * The quantized down-projection input is then the group-128 quantization of
 * the BF16 rounding of h (oracle_quantize_act on those BF16 values).
 */
void oracle_silu_mul(const uint16_t *gu, int64_t M, int64_t I, double *h)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t i = 0; i < I; i++) {
            double g = (double)bf16_bits_to_float(gu[m * 2 * I + i]);
            double u = (double)bf16_bits_to_float(gu[m * 2 * I + I + i]);
            h[m * I + i] = g / (1.0 + exp(-g)) * u;
        }
    }
}

/* oracle_bf16_round over an array. */
void oracle_bf16_round_array(const double *v, int64_t n, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_bf16_round(v[i]);
}

/*
 * NVFP4 weight-only format with BF16 activations (page
 * "ProCreations/Nanbeige4.3-33B-NVFP4-A16", the recipe paragraph: FP4 E2M1
 * weights in groups of 16 with E4M3 block scales and a global weight scale;
 * activations stay BF16).  A weight is
 *     w = e2m1(q) * e4m3(sb) * g
 * with q the 4-bit code, sb the E4M3 code of its 16-element group (16
 * consecutive k of one row) and g one FP32 scale per tensor.
 *
 * E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 */
double oracle_e2m1_decode(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* nearest E2M1 value, ties to the even mantissa, magnitudes above 6 -> 6 */
uint8_t oracle_e2m1_encode(float y)
{
    uint8_t sign = signbit(y) ? 0x8 : 0x0;
    double a = fabs((double)y);
    /* grid of the 8 magnitudes; between neighbours pick the nearer, ties to even m */
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    if (!(a < 6.0))
        return sign | 0x7; /* saturate (NaN is outside the contract) */
    int best = 0;
    for (int c = 1; c < 8; c++) {
        double d_best = fabs(a - mag[best]), d = fabs(a - mag[c]);
        if (d < d_best || (d == d_best && (c & 1) == 0 && (best & 1) == 1))
            best = c;
    }
    return sign | (uint8_t)best;
}

/*
 * Plain min-max NVFP4 quantization of W [N, K] (BF16 bits), the reading taken
 * here (the page's own scales come from a data-driven search, which needs
 * calibration data):
 *   g   = fl32(amax(W) / 2688)            (2688 = 6 * 448; 1 if W is all zero)
 *   sb  = E4M3_RNE_sat(fl32(amax_group / fl32(6 * g)))
 *   sig = fl32(e4m3(sb) * g)
 *   q   = E2M1_RNE_sat(fl32(w / sig))       (0 when sig is 0)
 * packed: [N, K/2] bytes, element 2j in the low nibble, 2j+1 in the high one;
 * sb: [N, K/16] E4M3 codes; *g_out: the global scale.
 */
void oracle_nvfp4_quantize(const uint16_t *w, int64_t N, int64_t K, uint8_t *packed, uint8_t *sb,
                           float *g_out)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < N * K; i++) {
        float a = fabsf(bf16_bits_to_float(w[i]));
        if (a > amax)
            amax = a;
    }
    float g = amax == 0.0f ? 1.0f : amax / 2688.0f;
    float six_g = 6.0f * g;
    *g_out = g;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < K / 16; b++) {
            const uint16_t *wb = w + n * K + b * 16;
            float ab = 0.0f;
            for (int i = 0; i < 16; i++) {
                float a = fabsf(bf16_bits_to_float(wb[i]));
                if (a > ab)
                    ab = a;
            }
            uint8_t code = oracle_e4m3_encode(ab / six_g);
            sb[n * (K / 16) + b] = code;
            float sig = (float)oracle_e4m3_decode(code) * g;
            for (int i = 0; i < 16; i += 2) {
                uint8_t lo = 0, hi = 0;
                if (sig != 0.0f) {
                    lo = oracle_e2m1_encode(bf16_bits_to_float(wb[i]) / sig);
                    hi = oracle_e2m1_encode(bf16_bits_to_float(wb[i + 1]) / sig);
                }
                packed[n * (K / 2) + (b * 16 + i) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/*
 * Y_ref[m, n] = sum_k x[m, k] * e2m1(q[n, k]) * e4m3(sb[n, k/16]) * g in FP64,
 * x BF16 [M, K]; rows of Y listed in `rows` (all when rows is NULL, n_rows = M).
 */
void oracle_nvfp4_gemm_ref(const uint16_t *x, const int64_t *rows, int64_t n_rows, int64_t K,
                           const uint8_t *packed, const uint8_t *sb, float g, int64_t N, double *y)
{
#pragma omp parallel
    {
        double *wr = (double *)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; n++) {
            for (int64_t k = 0; k < K; k++) {
                uint8_t byte = packed[n * (K / 2) + k / 2];
                uint8_t q = (k & 1) ? (byte >> 4) : (byte & 0xF);
                wr[k] = oracle_e2m1_decode(q) * oracle_e4m3_decode(sb[n * (K / 16) + k / 16]) *
                        (double)g;
            }
            for (int64_t r = 0; r < n_rows; r++) {
                int64_t m = rows ? rows[r] : r;
                const uint16_t *xm = x + m * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; k++)
                    acc += (double)bf16_bits_to_float(xm[k]) * wr[k];
                y[r * N + n] = acc;
            }
        }
        free(wr);
    }
}
