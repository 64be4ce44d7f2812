/*
 * CPU oracle for the LLM.int8() linear layer  --  TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package's smoke check and the bench's CPU-baseline leg
 * may load this library. The product path never calls it and shares no code,
 * header, table or helper with it.
 *
 * Plain, slow, single-threaded C, written step by step from the pages:
 *
 *   [P4] "LLM.int8() paper summary" (kurtkim.github.io/p/llm.int8/)
 *        - "8-bit Data Types and Quantization", absmax equation:
 *            X_i8 = round(127 / max|X| * X), range [-127, 127]
 *        - "Int8 Matrix Multiplication with 16-bit Float Inputs and Outputs":
 *            C ~= S * C_i32 = S * A_i8 B_i8, int32 accumulation
 *        - "Vector-wise Quantization": one scale per row of X and per output
 *            channel of W; dequantize by the outer product 1/(c_x (x) c_w)
 *        - "The Core of LLM.int8(): Mixed-precision Decomposition":
 *            C ~= sum_{h in O} X^h W^h (16-bit) + S * sum_{h not in O} X_i8^h W_i8^h,
 *            O = feature dims h holding a value of magnitude >= alpha = 6.0
 *   [P2] "Hugging Face LLM.int8() integration" (agentlenshq.com)
 *        - three-step recipe: extract outlier columns, vector-wise int8
 *          product of the rest, dequantize and add the fp16 outlier product
 *        - absmax worked example [1.2, -0.5, -4.3, ..., 5.4] -> scale 127/5.4
 *        - weights stored as int8 CB in [-127, 127] plus SCB, with
 *          W ~= CB * SCB / 127
 *
 * Readings where the pages are silent (each one also listed in the design
 * notes): outlier test is |x| >= threshold compared in fp32; the row scale of
 * X is the absmax over the NON-outlier columns only; the weight scale SCB_j is
 * the absmax over all K of output channel j; codes are rint(x * (127/absmax))
 * with both the division and the product rounded to fp32 and ties to even;
 * absmax 0 gives scale 0 and all-zero codes; when no fp16 outlier weight is
 * supplied the outlier weights are fp16(fp32(CB * SCB) / 127); the
 * dequantization, outlier product and bias are accumulated in fp64.
 *
 * fp16 values cross this interface as raw IEEE binary16 bit patterns
 * (uint16_t). The decoder and the round-to-nearest-even encoder below are
 * written from the IEEE 754 binary16 definition.
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * No FMA contraction and no fast-math, so every fp32 step rounds once.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- fp16 -- */

/* IEEE binary16 -> double, exact (every binary16 value is a double). */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (exp == 0) {
        v = ldexp((double)man, -24);               /* subnormal: man * 2^-24 */
    } else if (exp == 31) {
        v = man ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + man), exp - 25); /* (1.man) * 2^(exp-15) */
    }
    return sign ? -v : v;
}

/* double -> IEEE binary16, round to nearest, ties to even. */
uint16_t oracle_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7e00;
    if (a >= 65520.0) return sign | 0x7c00;        /* >= max + half ulp: inf */
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: units of 2^-24; 1024 units is the smallest normal,
         * whose encoding 0x0400 is exactly 1024, so no special case. */
        double r = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)r;
    }
    int e2;
    frexp(a, &e2);                                 /* a in [2^(e2-1), 2^e2) */
    int E = e2 - 1;
    double r = nearbyint(ldexp(a, 10 - E));        /* in [1024, 2048] */
    if (r >= 2048.0) { r = 1024.0; E += 1; }
    if (E + 15 >= 31) return sign | 0x7c00;
    return sign | (uint16_t)((E + 15) << 10) | (uint16_t)((int)r - 1024);
}

static float h2f(uint16_t h) { return (float)oracle_half_to_double(h); }

/* ------------------------------------------------ step 1: outlier set O -- */

/* [P2 step 1], [P4 mixed-precision decomposition]: O is the set of feature
 * columns h of X [M, K] holding any |X_ih| >= threshold. Writes O ascending
 * into idx (capacity K) and returns |O|. */
int64_t oracle_outlier_columns(const uint16_t *X, int64_t M, int64_t K,
                               float threshold, int32_t *idx)
{
    int64_t n = 0;
    for (int64_t h = 0; h < K; ++h) {
        int hit = 0;
        for (int64_t i = 0; i < M && !hit; ++i) {
            float ax = fabsf(h2f(X[i * K + h]));
            if (ax >= threshold) hit = 1;
        }
        if (hit) idx[n++] = (int32_t)h;
    }
    return n;
}

/* ------------------------------------------- step 2: absmax quantization -- */

/* [P4 absmax equation] applied to one vector: scale by 127/absmax (fp32
 * division), multiply (fp32), round to nearest integer (ties to even),
 * clamp to [-127, 127]. mask[h] != 0 excludes element h (code 0, not part of
 * the absmax). Returns the absmax (the stored scale). */
static float quantize_vector(const uint16_t *x, const unsigned char *mask,
                             int64_t n, int8_t *q)
{
    float absmax = 0.0f;
    for (int64_t h = 0; h < n; ++h) {
        if (mask && mask[h]) continue;
        float a = fabsf(h2f(x[h]));
        if (a > absmax) absmax = a;
    }
    if (absmax == 0.0f) {
        for (int64_t h = 0; h < n; ++h) q[h] = 0;
        return 0.0f;
    }
    float s = 127.0f / absmax;
    for (int64_t h = 0; h < n; ++h) {
        if (mask && mask[h]) { q[h] = 0; continue; }
        float p = h2f(x[h]) * s;
        float r = nearbyintf(p);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[h] = (int8_t)r;
    }
    return absmax;
}

/* [P2 step 2], [P4 vector-wise quantization]: X rows, one scale per row over
 * the non-outlier columns; outlier columns get code 0. Also returns O. */
int64_t oracle_quantize_rows(const uint16_t *X, int64_t M, int64_t K, float threshold,
                             int8_t *CA, float *SCA, int32_t *outlier_idx)
{
    int64_t n_out = oracle_outlier_columns(X, M, K, threshold, outlier_idx);
    unsigned char *mask = (unsigned char *)calloc((size_t)K, 1);
    for (int64_t t = 0; t < n_out; ++t) mask[outlier_idx[t]] = 1;
    for (int64_t i = 0; i < M; ++i)
        SCA[i] = quantize_vector(X + i * K, mask, K, CA + i * K);
    free(mask);
    return n_out;
}

/* [P2 transformers integration]: weights W [N, K] become int8 CB in
 * [-127, 127] with one scale SCB_j per output channel j (absmax over all K),
 * so that W ~= CB * SCB / 127. */
void oracle_prepare_weight(const uint16_t *W, int64_t N, int64_t K, int8_t *CB, float *SCB)
{
    for (int64_t j = 0; j < N; ++j)
        SCB[j] = quantize_vector(W + j * K, NULL, K, CB + j * K);
}

/* ---------------------------------------------- step 3: int8 GEMM, int32 -- */

/* [P4 int8 matmul equation]: C_ij = sum_k A_ik * B_jk with int32 result.
 * Accumulated in int64; returns 0, or -1 if some C_ij does not fit int32. */
int oracle_gemm_i32(const int8_t *A, const int8_t *B, int64_t M, int64_t N, int64_t K,
                    int32_t *C)
{
    int ok = 0;
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < N; ++j) {
            int64_t acc = 0;
            const int8_t *a = A + i * K, *b = B + j * K;
            for (int64_t k = 0; k < K; ++k) acc += (int64_t)a[k] * (int64_t)b[k];
            if (acc > INT32_MAX || acc < INT32_MIN) ok = -1;
            C[i * N + j] = (int32_t)acc;
        }
    return ok;
}

/* ------------------------------------- steps 4-5: dequantize and combine -- */

/* The fp16 outlier weight of channel j, feature h. [P4 decomposition] uses the
 * fp16 weight W^h. When only the int8 weights are kept, the [P2] recovery
 * CB * SCB / 127 stands in for it (fp32 product and division, then fp16). */
static double outlier_weight(const uint16_t *W_outlier, const int8_t *CB, const float *SCB,
                             int64_t K, int64_t j, int64_t h)
{
    if (W_outlier) return oracle_half_to_double(W_outlier[j * K + h]);
    float t = (float)CB[j * K + h] * SCB[j];
    float u = t / 127.0f;
    return oracle_half_to_double(oracle_double_to_half((double)u));
}

/* Full forward for selected output rows ("rows", nrows) and all N columns:
 *   Y_ij = C_ij * SCA_i * SCB_j / 127^2              [P4 vector-wise eq.]
 *        + sum_{h in O} X_ih * Wo_jh                 [P4 decomposition]
 *        + bias_j
 * in fp64 (Y64) and rounded to fp16 (Y16, may be NULL). CA/SCA are quantized
 * here from X; CB/SCB are given (from oracle_prepare_weight). Returns |O|,
 * or -1 if an int32 accumulator overflowed. */
int64_t oracle_forward_rows(const uint16_t *X, int64_t M, int64_t N, int64_t K,
                            const int8_t *CB, const float *SCB, const uint16_t *W_outlier,
                            float threshold, const uint16_t *bias,
                            const int64_t *rows, int64_t nrows,
                            double *Y64, uint16_t *Y16)
{
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
    int8_t *ca = (int8_t *)malloc((size_t)(K > 0 ? K : 1));
    unsigned char *mask = (unsigned char *)calloc((size_t)(K > 0 ? K : 1), 1);
    int64_t n_out = oracle_outlier_columns(X, M, K, threshold, idx);
    int overflow = 0;
    for (int64_t t = 0; t < n_out; ++t) mask[idx[t]] = 1;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows[r];
        const uint16_t *xrow = X + i * K;
        float sca = quantize_vector(xrow, mask, K, ca);
        for (int64_t j = 0; j < N; ++j) {
            int64_t acc = 0;
            const int8_t *b = CB + j * K;
            for (int64_t k = 0; k < K; ++k) acc += (int64_t)ca[k] * (int64_t)b[k];
            if (acc > INT32_MAX || acc < INT32_MIN) overflow = 1;
            double y = (double)acc * (double)sca * (double)SCB[j] / 16129.0;
            for (int64_t t = 0; t < n_out; ++t) {
                int64_t h = idx[t];
                y += oracle_half_to_double(xrow[h]) *
                     outlier_weight(W_outlier, CB, SCB, K, j, h);
            }
            if (bias) y += oracle_half_to_double(bias[j]);
            Y64[r * N + j] = y;
            if (Y16) Y16[r * N + j] = oracle_double_to_half(y);
        }
    }
    free(idx);
    free(ca);
    free(mask);
    return overflow ? -1 : n_out;
}

/* All rows. */
int64_t oracle_forward(const uint16_t *X, int64_t M, int64_t N, int64_t K,
                       const int8_t *CB, const float *SCB, const uint16_t *W_outlier,
                       float threshold, const uint16_t *bias, double *Y64, uint16_t *Y16)
{
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(M > 0 ? M : 1));
    for (int64_t i = 0; i < M; ++i) rows[i] = i;
    int64_t r = oracle_forward_rows(X, M, N, K, CB, SCB, W_outlier, threshold, bias,
                                    rows, M, Y64, Y16);
    free(rows);
    return r;
}

/* The fp16 outlier weights as the layer uses them, gathered: Wo[j, t] for
 * t < |O| (same rule as the forward). For tests of the gather step. */
void oracle_outlier_weights(const uint16_t *W_outlier, const int8_t *CB, const float *SCB,
                            int64_t N, int64_t K, const int32_t *idx, int64_t n_out,
                            uint16_t *Wo)
{
    for (int64_t j = 0; j < N; ++j)
        for (int64_t t = 0; t < n_out; ++t)
            Wo[j * n_out + t] =
                oracle_double_to_half(outlier_weight(W_outlier, CB, SCB, K, j, idx[t]));
}

/* ------------------------------------ zeropoint (asymmetric) quantization -- */

/* [P4 "8-bit Data Types and Quantization", zeropoint quantization] applied to
 * one vector. The normalized dynamic range nd = 2*127 / (max - min) scales the
 * vector; the zeropoint zp shifts it so that it spans [-127, 127]. The page's
 * zp formula is garbled ("X * min X"); the reading taken: zp = rint(nd * min)
 * + 127 and X_i8 = clamp(rint(nd * X) - zp, -127, 127), so that
 * X ~= (X_i8 + zp) / nd, which is the form the page's product
 * (A_i8 + zp_a)(B_i8 + zp_b) uses. fp32 steps as for absmax: nd is the fp32
 * quotient of 254 by the fp32 difference max - min; products are fp32; rint
 * rounds ties to even. A constant vector (max == min) takes nd = 1.
 * Returns nd; *zp gets the zeropoint and *sum the sum of the codes. */
static float zp_quantize_vector(const uint16_t *x, int64_t n, int8_t *q, int32_t *zp, int32_t *sum)
{
    float mn = INFINITY, mx = -INFINITY;
    for (int64_t h = 0; h < n; ++h) {
        float v = h2f(x[h]);
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    if (n == 0) mn = mx = 0.0f;
    float range = mx - mn;
    float nd = range > 0.0f ? 254.0f / range : 1.0f;
    float zmin = nearbyintf(mn * nd);   /* |nd * min| <= 254 * 2^10: exact in fp32 and int32 */
    int32_t z = (int32_t)zmin + 127;
    int64_t s = 0;
    for (int64_t h = 0; h < n; ++h) {
        int64_t c = (int64_t)nearbyintf(h2f(x[h]) * nd) - z;
        if (c > 127) c = 127;
        if (c < -127) c = -127;
        q[h] = (int8_t)c;
        s += c;
    }
    *zp = z;
    *sum = (int32_t)s;
    return nd;
}

/* Zeropoint quantization of every row of an fp16 matrix [R, K] (the tokens
 * of X, or the output channels of W): codes, nd, zp and the code sums. */
void oracle_zp_quantize_rows(const uint16_t *X, int64_t R, int64_t K, int8_t *Q, float *ND,
                             int32_t *ZP, int32_t *SUM)
{
    for (int64_t i = 0; i < R; ++i) ND[i] = zp_quantize_vector(X + i * K, K, Q + i * K, ZP + i, SUM + i);
}

/* Forward with zeropoint quantization on both sides, no outlier split, for
 * selected rows of X:
 *   C_ij = (A_i + zp_a_i) . (B_j + zp_b_j)                         [P4]
 *        = A_i . B_j + zp_b_j * sum(A_i) + zp_a_i * sum(B_j) + K zp_a_i zp_b_j
 * (the page's unrolled form, in int64: the first term is the int8 GEMM, the
 * other three are the corrections), Y_ij = C_ij / (nd_a_i nd_b_j) + bias_j
 * in fp64. CB, NDB, ZPB, SUMB come from oracle_zp_quantize_rows on W. */
void oracle_zp_forward_rows(const uint16_t *X, int64_t M, int64_t N, int64_t K,
                            const int8_t *CB, const float *NDB, const int32_t *ZPB, const int32_t *SUMB,
                            const uint16_t *bias, const int64_t *rows, int64_t nrows, double *Y64)
{
    int8_t *ca = (int8_t *)malloc((size_t)(K > 0 ? K : 1));
    (void)M;
    for (int64_t r = 0; r < nrows; ++r) {
        int32_t za, sa;
        float nda = zp_quantize_vector(X + rows[r] * K, K, ca, &za, &sa);
        for (int64_t j = 0; j < N; ++j) {
            int64_t dot = 0;
            const int8_t *b = CB + j * K;
            for (int64_t k = 0; k < K; ++k) dot += (int64_t)ca[k] * (int64_t)b[k];
            int64_t c = dot + (int64_t)ZPB[j] * sa + (int64_t)za * SUMB[j] + K * (int64_t)za * ZPB[j];
            double y = (double)c / ((double)nda * (double)NDB[j]);
            if (bias) y += oracle_half_to_double(bias[j]);
            Y64[r * N + j] = y;
        }
    }
    free(ca);
}
