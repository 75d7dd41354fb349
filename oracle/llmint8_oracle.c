/*
 * CPU oracle for the LLM.int8() mixed-precision decomposed linear layer  Y = X . W^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this
 * file; only the test suite, the package's smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * It is the plain definition of the method, written out step by step in the order the
 * pages give it, with no blocking, fusion or reordering:
 *
 *   "A gentle introduction to 8-bit matrix multiplication for transformers at scale"
 *   (Hugging Face blog, zh translation), sections "模型量化介绍" (absmax quantization and
 *   its worked example; vector-wise quantization with an outer-product dequantization),
 *   "LLM.int8() 温和总结" (the three steps), "MatMul 内部" (threshold 6: magnitude 6 or
 *   more; hidden states quantized by row, weights by column), "用法" (int8 weights CB,
 *   per-channel statistic SCB, dequantization (CB * SCB) / 127).
 *
 *   "LLM.int8(): 8-Bit Matrix Multiplication for Transformers at Scale" (azimuth.plus
 *   summary of Dettmers et al., NeurIPS 2022), sections "الابتكار الأول" (vector-wise
 *   quantization), "الابتكار الثاني" (mixed-precision decomposition) and "الصورة الكاملة"
 *   (the four-stage method: find outlier feature columns, split X and W along them,
 *   fp16 product of the outlier part, int8 product of the rest dequantized by the outer
 *   product of the scale vectors, sum in 16 bit).
 *
 * Readings taken where the pages are silent (each is listed with its reason in the
 * design notes of the repository):
 *   - a column of X is an outlier when ANY of its entries has |x| >= threshold;
 *   - the row absmax of X is taken over the NON-outlier columns only (decompose first,
 *     then quantize the regular part);
 *   - the stored statistics are the absmax values (fp32); the quantization multiplier is
 *     fl32(127 / absmax); q = round-half-to-even(fl32(x * multiplier)), clamped to
 *     [-127, 127]; a row whose absmax is 0 quantizes to all zeros;
 *   - the fp16 weights of the outlier columns are the dequantized ones,
 *     fp16(fl32(fl32(CB * SCB) / 127)), unless the caller supplies the original fp16 W;
 *   - the final sum C * SCA * SCB / 127^2 + sum_outliers X * W_o + bias is evaluated in
 *     fp64 and rounded once to fp16 (round-half-to-even).
 *
 * fp32 steps use C `float` arithmetic (IEEE binary32, round to nearest even; build with
 * -ffp-contract=off so no multiply is fused).  fp16 values are passed as their raw
 * uint16_t bit patterns and decoded/encoded here from the IEEE binary16 definition.
 *
 * Status codes: 0 = ok, 1 = invalid argument, 4 = outlier capacity exceeded,
 * 7 = an int32 accumulator would overflow.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_INVALID_ARG 1
#define ORACLE_ERR_OUTLIER_CAPACITY 4
#define ORACLE_ERR_INT32_OVERFLOW 7

/* ---------------------------------------------------------------- binary16 ---------- */

/* Exact value of an IEEE binary16 bit pattern. */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);     /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Round a double to the nearest binary16 value, ties to even. */
uint16_t oracle_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x))
        return 0x7e00;
    /* largest finite half is 65504; the midpoint to the next step (65536) is 65520 */
    if (a >= 65520.0)
        return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: a multiple of 2^-24; 1024 * 2^-24 is the smallest normal,
           whose encoding 0x0400 follows on from the subnormal codes */
        double q = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)q;
    }
    int e2;
    frexp(a, &e2);                 /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                /* a in [2^E, 2^(E+1)) */
    double q = nearbyint(ldexp(a, 10 - E));   /* significand scaled to [1024, 2048] */
    uint32_t mant = (uint32_t)q;
    if (mant == 2048) {
        mant = 1024;
        E += 1;
    }
    if (E > 15)
        return sign | 0x7c00;
    return sign | (uint16_t)((E + 15) << 10) | (uint16_t)(mant - 1024);
}

/* fp16 -> fp32 is exact. */
static float half_to_float(uint16_t h) { return (float)oracle_half_to_double(h); }

/* ------------------------------------------------------------ absmax step ---------- */

/* Absmax quantization of one value with the multiplier s = fl32(127 / absmax):
   q = round_half_even(fl32(x * s)), clamped to the symmetric int8 range. */
static int8_t absmax_quantize(float x, float s)
{
    float scaled = x * s;
    float r = nearbyintf(scaled);  /* default rounding mode: to nearest, ties to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* ----------------------------------------------- weights: one scale per output row ---- */

/* W fp16 [N, K] row-major (row n = output channel n, K contiguous).
   SCB[n] = max_k |W[n, k]|;  CB[n, k] = q(W[n, k], fl32(127 / SCB[n])).
   (The blog quantizes the weight per column of the logical K x N weight, which is per
   output channel: per row of CB.) */
int oracle_quantize_weight_colwise(const uint16_t *W, int64_t N, int64_t K,
                                   int8_t *CB, float *SCB)
{
    if (!W || !CB || !SCB || N < 1 || K < 1)
        return ORACLE_ERR_INVALID_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *w = W + n * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(half_to_float(w[k]));
            if (v > amax) amax = v;
        }
        SCB[n] = amax;
        int8_t *cb = CB + n * K;
        if (amax == 0.0f) {
            memset(cb, 0, (size_t)K);
            continue;
        }
        float s = 127.0f / amax;
        for (int64_t k = 0; k < K; ++k)
            cb[k] = absmax_quantize(half_to_float(w[k]), s);
    }
    return ORACLE_OK;
}

/* ----------------------------------- activations: outlier columns, then rows ---------- */

/* Step 1: column j of X is an outlier feature when some row has |X[i, j]| >= threshold.
   is_outlier[j] receives 0/1. */
static void find_outlier_columns(const uint16_t *X, int64_t M, int64_t K, float threshold,
                                 unsigned char *is_outlier)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < K; ++j) {
        unsigned char flag = 0;
        for (int64_t i = 0; i < M; ++i) {
            if (fabsf(half_to_float(X[i * K + j])) >= threshold) {
                flag = 1;
                break;
            }
        }
        is_outlier[j] = flag;
    }
}

/* Steps 2-3 for one row: absmax over the regular (non-outlier) columns, then absmax
   quantization of the regular part; outlier columns hold 0 in Xq. */
static void quantize_row(const uint16_t *x, int64_t K, const unsigned char *is_outlier,
                         int8_t *xq, float *sca)
{
    float amax = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
        if (is_outlier[j]) continue;
        float v = fabsf(half_to_float(x[j]));
        if (v > amax) amax = v;
    }
    *sca = amax;
    if (amax == 0.0f) {
        memset(xq, 0, (size_t)K);
        return;
    }
    float s = 127.0f / amax;
    for (int64_t j = 0; j < K; ++j)
        xq[j] = is_outlier[j] ? 0 : absmax_quantize(half_to_float(x[j]), s);
}

/* X fp16 [M, K].  Writes Xq int8 [M, K], SCA fp32 [M], the ascending outlier column list
   (at most `cap` entries) and its true length in *n_outliers. */
int oracle_quantize_rows_and_find_outliers(const uint16_t *X, int64_t M, int64_t K,
                                           float threshold, int8_t *Xq, float *SCA,
                                           int32_t *outlier_idx, int32_t *n_outliers,
                                           int64_t cap)
{
    if (!X || !Xq || !SCA || !n_outliers || M < 1 || K < 1 || cap < 0 || isnan(threshold))
        return ORACLE_ERR_INVALID_ARG;
    unsigned char *is_outlier = (unsigned char *)malloc((size_t)K);
    if (!is_outlier) return ORACLE_ERR_INVALID_ARG;
    find_outlier_columns(X, M, K, threshold, is_outlier);
    int64_t count = 0;
    for (int64_t j = 0; j < K; ++j) {
        if (!is_outlier[j]) continue;
        if (count < cap && outlier_idx) outlier_idx[count] = (int32_t)j;
        ++count;
    }
    *n_outliers = (int32_t)count;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i)
        quantize_row(X + i * K, K, is_outlier, Xq + i * K, SCA + i);
    free(is_outlier);
    return count > cap ? ORACLE_ERR_OUTLIER_CAPACITY : ORACLE_OK;
}

/* ----------------------------------------------------------- int8 product ---------- */

/* C[i, n] = sum_k Xq[i, k] * CB[n, k], exact in int64, checked to fit int32. */
int oracle_int8_accumulate(const int8_t *Xq, int64_t M, int64_t K, const int8_t *CB,
                           int64_t N, int32_t *C)
{
    if (!Xq || !CB || !C || M < 1 || K < 1 || N < 1)
        return ORACLE_ERR_INVALID_ARG;
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k)
                acc += (int64_t)Xq[i * K + k] * (int64_t)CB[n * K + k];
            if (acc > INT32_MAX || acc < INT32_MIN) overflow = 1;
            C[i * N + n] = (int32_t)acc;
        }
    }
    return overflow ? ORACLE_ERR_INT32_OVERFLOW : ORACLE_OK;
}

/* ------------------------------------------------------------- dequant ------------- */

/* W_hat[n, k] = fp16(fl32(fl32(CB[n, k] * SCB[n]) / 127)), evaluated in that order. */
static float dequant_value(int8_t cb, float scb)
{
    float prod = (float)cb * scb;
    return prod / 127.0f;
}

int oracle_dequant(const int8_t *CB, const float *SCB, int64_t N, int64_t K, uint16_t *W_out)
{
    if (!CB || !SCB || !W_out || N < 1 || K < 1)
        return ORACLE_ERR_INVALID_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            W_out[n * K + k] = oracle_double_to_half((double)dequant_value(CB[n * K + k], SCB[n]));
    return ORACLE_OK;
}

/* ------------------------------------------------------------ full layer ----------- */

/* The fp16 weight of outlier column j for output n: the dequantized int8 weight, or the
   original fp16 weight when the caller keeps it. */
static double outlier_weight(const int8_t *CB, const float *SCB, const uint16_t *W_fp16,
                             int64_t K, int64_t n, int64_t j)
{
    if (W_fp16)
        return oracle_half_to_double(W_fp16[n * K + j]);
    uint16_t h = oracle_double_to_half((double)dequant_value(CB[n * K + j], SCB[n]));
    return oracle_half_to_double(h);
}

/* Output element (i, n):  fp16( C*SCA_i*SCB_n/127^2 + sum_{j in O} X[i,j]*W_o[n,j] + bias_n )
   with the sum evaluated in fp64. */
static uint16_t output_element(const uint16_t *X, int64_t K, const int8_t *CB,
                               const float *SCB, const uint16_t *bias,
                               const uint16_t *W_fp16, const int32_t *O, int64_t nO,
                               const int8_t *Xq, const float *SCA, int64_t i, int64_t n,
                               int32_t *c_out, int *overflow)
{
    int64_t acc = 0;
    for (int64_t k = 0; k < K; ++k)
        acc += (int64_t)Xq[i * K + k] * (int64_t)CB[n * K + k];
    if (acc > INT32_MAX || acc < INT32_MIN) *overflow = 1;
    if (c_out) *c_out = (int32_t)acc;
    double y = (double)acc * (double)SCA[i] * (double)SCB[n] / 16129.0;
    for (int64_t t = 0; t < nO; ++t) {
        int64_t j = O[t];
        y += oracle_half_to_double(X[i * K + j]) * outlier_weight(CB, SCB, W_fp16, K, n, j);
    }
    if (bias) y += oracle_half_to_double(bias[n]);
    return oracle_double_to_half(y);
}

/* Full layer on host arrays.  X fp16 [M, K]; CB int8 [N, K]; SCB fp32 [N];
   bias fp16 [N] or NULL; W_fp16 fp16 [N, K] or NULL; Y fp16 [M, N];
   C_out int32 [M, N] or NULL (the int8 accumulators). */
int oracle_linear(const uint16_t *X, int64_t M, int64_t K, const int8_t *CB, const float *SCB,
                  int64_t N, const uint16_t *bias, const uint16_t *W_fp16, float threshold,
                  uint16_t *Y, int32_t *C_out)
{
    if (!X || !CB || !SCB || !Y || M < 1 || K < 1 || N < 1 || isnan(threshold))
        return ORACLE_ERR_INVALID_ARG;
    int8_t *Xq = (int8_t *)malloc((size_t)(M * K));
    float *SCA = (float *)malloc((size_t)M * sizeof(float));
    int32_t *O = (int32_t *)malloc((size_t)K * sizeof(int32_t));
    if (!Xq || !SCA || !O) { free(Xq); free(SCA); free(O); return ORACLE_ERR_INVALID_ARG; }
    int32_t nO = 0;
    oracle_quantize_rows_and_find_outliers(X, M, K, threshold, Xq, SCA, O, &nO, K);
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t n = 0; n < N; ++n)
            Y[i * N + n] = output_element(X, K, CB, SCB, bias, W_fp16, O, nO, Xq, SCA, i, n,
                                          C_out ? C_out + i * N + n : NULL, &overflow);
    free(Xq); free(SCA); free(O);
    return overflow ? ORACLE_ERR_INT32_OVERFLOW : ORACLE_OK;
}

/* Same definition, evaluated only at the listed (rows[s], cols[s]) output positions, for
   shapes whose full product is too large for a plain CPU loop.  The outlier set and the
   row quantization always cover all of X, as the definition requires. */
int oracle_linear_sampled(const uint16_t *X, int64_t M, int64_t K, const int8_t *CB,
                          const float *SCB, int64_t N, const uint16_t *bias,
                          const uint16_t *W_fp16, float threshold, int64_t n_samples,
                          const int64_t *rows, const int64_t *cols, uint16_t *Y_out,
                          int32_t *C_out)
{
    if (!X || !CB || !SCB || !rows || !cols || !Y_out || M < 1 || K < 1 || N < 1 ||
        n_samples < 0 || isnan(threshold))
        return ORACLE_ERR_INVALID_ARG;
    for (int64_t s = 0; s < n_samples; ++s)
        if (rows[s] < 0 || rows[s] >= M || cols[s] < 0 || cols[s] >= N)
            return ORACLE_ERR_INVALID_ARG;
    int8_t *Xq = (int8_t *)malloc((size_t)(M * K));
    float *SCA = (float *)malloc((size_t)M * sizeof(float));
    int32_t *O = (int32_t *)malloc((size_t)K * sizeof(int32_t));
    if (!Xq || !SCA || !O) { free(Xq); free(SCA); free(O); return ORACLE_ERR_INVALID_ARG; }
    int32_t nO = 0;
    oracle_quantize_rows_and_find_outliers(X, M, K, threshold, Xq, SCA, O, &nO, K);
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t s = 0; s < n_samples; ++s)
        Y_out[s] = output_element(X, K, CB, SCB, bias, W_fp16, O, nO, Xq, SCA, rows[s], cols[s],
                                  C_out ? C_out + s : NULL, &overflow);
    free(Xq); free(SCA); free(O);
    return overflow ? ORACLE_ERR_INT32_OVERFLOW : ORACLE_OK;
}
