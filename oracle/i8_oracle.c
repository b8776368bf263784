/*
 * i8_oracle.c -- plain, slow CPU oracle for the LLM.int8() decomposed linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the test-suite, the smoke check and the CPU-baseline leg of the benchmark
 * do.  It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (all from the pages "A Gentle Introduction to 8-bit Matrix Multiplication for
 * transformers at scale" (Hugging Face blog, Chinese translation), its summary on
 * agentlenshq.com, and the LLM.int8() abstract):
 *   - absmax quantisation: scale = 127 / max|x|, code = round(x * scale)
 *     ("absmax 量化", the [1.2, -0.5, ..., 5.4] worked example);
 *   - vector-wise quantisation: one absmax per row of the hidden states and one per
 *     output channel of the weight, dequantised by the outer product of the two absmax
 *     vectors ("absmax 量化", the A*B=C paragraph; "内部的 MatMul");
 *   - the three-step decomposition: outlier columns of the hidden states are found with
 *     a threshold, multiplied in fp16, the rest in int8, and the two results are added
 *     ("LLM.int8() 的总结"; "内部的 MatMul": magnitude 6 or larger);
 *   - weight recovery for the outlier product: CB * SCB / 127 ("用法", the printout
 *     after .to(0)).
 *
 * Readings taken where the pages are silent (each listed in the design notes):
 *   - an element is an outlier when |x| >= threshold ("6 or larger");
 *   - a column is an outlier column when any row of the call has an outlier in it;
 *   - the row absmax of X runs over the non-outlier columns only; the weight absmax
 *     runs over the whole output row (per output channel);
 *   - rounding is half away from zero (C99 roundf), applied to the fp32 product
 *     x * fl32(127 / absmax); a zero absmax gives scale 0 and all-zero codes;
 *   - the reference output is formed in fp64 (no fp16 rounding of the result).
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fPIC -shared (see build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* IEEE 754 binary16 -> binary32 by the format's definition: 1 sign bit, 5 exponent
 * bits (bias 15), 10 fraction bits; exponent 0 is zero/subnormal (value f * 2^-24),
 * exponent 31 is inf/NaN.  Every binary16 value is exact in binary32. */
float oracle_half_to_float(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    float v;
    if (e == 0) {
        v = ldexpf((float)f, -24);
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexpf((float)(f + 1024), e - 25);
    }
    return sign ? -v : v;
}

/* Step 1 -- outlier column scan.  is_outlier[k] = 1 when some row t has
 * |X[t,k]| >= threshold.  idx receives the outlier columns in ascending order and
 * *n_o their count.  mask_words (nullable) receives the same set packed 32 columns per
 * word, column k at bit (k % 32) of word k / 32. */
void oracle_outlier_scan(const uint16_t *X, int64_t T, int64_t K, float threshold,
                         uint8_t *is_outlier, uint32_t *mask_words,
                         int32_t *idx, int32_t *n_o)
{
    for (int64_t k = 0; k < K; ++k)
        is_outlier[k] = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t k = 0; k < K; ++k)
            if (fabsf(oracle_half_to_float(X[t * K + k])) >= threshold)
                is_outlier[k] = 1;
    int32_t count = 0;
    for (int64_t k = 0; k < K; ++k)
        if (is_outlier[k])
            idx[count++] = (int32_t)k;
    *n_o = count;
    if (mask_words) {
        int64_t words = (K + 31) / 32;
        for (int64_t w = 0; w < words; ++w)
            mask_words[w] = 0;
        for (int64_t k = 0; k < K; ++k)
            if (is_outlier[k])
                mask_words[k / 32] |= (uint32_t)1 << (k % 32);
    }
}

/* Steps 2 and 3 -- row-wise absmax quantisation of an fp16 matrix A [R,K].
 * skip (nullable) marks columns excluded from the absmax and coded as 0 (the outlier
 * columns of the hidden states; NULL for the weight, whose scale covers the whole
 * output row).  scale[r] = max |A[r,k]| over the kept columns, as fp32;
 * q[r,k] = round_half_away(fl32(A[r,k] * fl32(127 / scale[r]))). */
void oracle_absmax_quantize_rows(const uint16_t *A, int64_t R, int64_t K,
                                 const uint8_t *skip, int8_t *q, float *scale)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        const uint16_t *row = A + r * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (skip && skip[k])
                continue;
            float a = fabsf(oracle_half_to_float(row[k]));
            if (a > amax)
                amax = a;
        }
        scale[r] = amax;
        int8_t *qr = q + r * K;
        if (amax == 0.0f) {
            for (int64_t k = 0; k < K; ++k)
                qr[k] = 0;
            continue;
        }
        float s = 127.0f / amax;
        for (int64_t k = 0; k < K; ++k) {
            if (skip && skip[k]) {
                qr[k] = 0;
                continue;
            }
            float v = oracle_half_to_float(row[k]) * s;
            float c = roundf(v);
            if (c > 127.0f) c = 127.0f;
            if (c < -127.0f) c = -127.0f;
            qr[k] = (int8_t)c;
        }
    }
}

/* Step 4 -- integer matmul acc[i,n] = sum_k A[rows[i],k] * B[n,k] (B in the
 * [out,in] layout), accumulated in int64 and returned as int32.  rows (nullable)
 * selects a subset of A's rows; otherwise rows 0..nrows-1.  Returns the number of
 * results that do not fit in int32 (0 at every size the layer admits). */
int64_t oracle_int_matmul(const int8_t *A, const int8_t *B, int64_t nrows,
                          const int64_t *rows, int64_t N, int64_t K, int32_t *acc)
{
    int64_t overflow = 0;
    #pragma omp parallel for collapse(2) schedule(static) reduction(+:overflow)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            const int8_t *a = A + (rows ? rows[i] : i) * K;
            const int8_t *b = B + n * K;
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)a[k] * (int64_t)b[k];
            if (s > INT32_MAX || s < INT32_MIN)
                ++overflow;
            acc[i * N + n] = (int32_t)s;
        }
    }
    return overflow;
}

/* Steps 5 and 6 -- the decomposed product for the selected rows, in fp64:
 *   C[i,n] = acc[i,n] * SCx[t] * SCB[n] / 127^2                  (int8 part, dequantised)
 *          + sum_{j < n_o} X[t, idx[j]] * CB[n, idx[j]] * SCB[n] / 127   (fp16 outlier part)
 *          + bias[n]                                               (bias nullable)
 * with t = rows[i].  acc holds the int8 products of exactly those rows. */
void oracle_decomposed_output(const uint16_t *X, int64_t K, const int64_t *rows,
                              int64_t nrows, const int32_t *acc, const float *SCx,
                              const int8_t *CB, const float *SCB, const uint16_t *bias,
                              int64_t N, const int32_t *idx, int32_t n_o, double *C)
{
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t t = rows ? rows[i] : i;
            double int_part = (double)acc[i * N + n] * (double)SCx[t] * (double)SCB[n]
                              / (127.0 * 127.0);
            double out_part = 0.0;
            for (int32_t j = 0; j < n_o; ++j) {
                int64_t k = idx[j];
                double w = (double)CB[n * K + k] * (double)SCB[n] / 127.0;
                out_part += (double)oracle_half_to_float(X[t * K + k]) * w;
            }
            double b = bias ? (double)oracle_half_to_float(bias[n]) : 0.0;
            C[i * N + n] = int_part + out_part + b;
        }
    }
}

/* The whole forward for a subset of rows: steps 1 and 2 over ALL rows of X (the
 * column mask depends on every row of the call), then steps 4-6 for the selected rows
 * against an already-quantised weight (CB, SCB).  All outputs are caller-owned:
 * mask_words [ceil(K/32)], idx [K], n_o [1], Xq [T,K], SCx [T],
 * acc [nrows,N], C [nrows,N]. */
int64_t oracle_linear_forward_rows(const uint16_t *X, int64_t T, int64_t K,
                                   const int8_t *CB, const float *SCB,
                                   const uint16_t *bias, int64_t N, float threshold,
                                   const int64_t *rows, int64_t nrows,
                                   uint32_t *mask_words, int32_t *idx, int32_t *n_o,
                                   int8_t *Xq, float *SCx, int32_t *acc, double *C)
{
    uint8_t *is_outlier = (uint8_t *)malloc((size_t)(K > 0 ? K : 1));
    if (!is_outlier)
        return -1;
    oracle_outlier_scan(X, T, K, threshold, is_outlier, mask_words, idx, n_o);
    oracle_absmax_quantize_rows(X, T, K, is_outlier, Xq, SCx);
    int64_t overflow = oracle_int_matmul(Xq, CB, nrows, rows, N, K, acc);
    oracle_decomposed_output(X, K, rows, nrows, acc, SCx, CB, SCB, bias, N, idx, *n_o, C);
    free(is_outlier);
    return overflow;
}

/* ---------------------------------------------------------------------------------
 * FP8 (e4m3) variant of the decomposition.  The pages name 8-bit floating point only as
 * the next step ("LLM.int8() 的总结" / the closing outlook); the plainest reading keeps
 * every step above and swaps the int8 absmax code for an e4m3 code of the same scaled
 * value: scale = fl32(448 / absmax) (448 is the largest finite e4m3 magnitude, as 127 is
 * the largest int8 code used), code = e4m3 rounding of fl32(x * scale), and 448 in place
 * of 127 in every dequantisation (acc * SCx * SCB / 448^2, weights CB * SCB / 448).
 *
 * e4m3 is the "fn" format of the OCP 8-bit floating-point specification: 1 sign bit,
 * 4 exponent bits (bias 7), 3 fraction bits; exponent field 0 holds zero and the
 * subnormals (fraction * 2^-9); S.1111.111 is NaN; there are no infinities, and the
 * largest finite magnitude is 1.75 * 2^8 = 448. */

/* Decode one e4m3 code to its exact value. */
double oracle_e4m3_to_double(uint8_t c)
{
    int e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* Encode: round to the nearest e4m3 value, ties to the even fraction; magnitudes of 448
 * and above give 448 (round-to-nearest already does below 464, the midpoint to the next
 * power-of-two step; the scaled values of this layer never exceed 448 * (1 + 2^-23)). */
uint8_t oracle_e4m3_from_float(float v)
{
    if (isnan(v))
        return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0)
        return sign | 0x7E;
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);                    /* a in [2^(e-1), 2^e) */
    int E = e - 1;
    if (E < -6)
        E = -6;                      /* subnormals share the 2^-6 binade's step */
    double step = ldexp(1.0, E - 3); /* three fraction bits */
    double r = nearbyint(a / step) * step;   /* default rounding: nearest, ties to even */
    if (r == 0.0)
        return sign;
    int e2;
    frexp(r, &e2);
    int E2 = e2 - 1;
    if (E2 < -6)
        return sign | (uint8_t)(r / ldexp(1.0, -9));
    int m = (int)((ldexp(r, -E2) - 1.0) * 8.0);
    return sign | (uint8_t)(((E2 + 7) << 3) | m);
}

/* Row-wise absmax e4m3 quantisation of an fp16 matrix A [R,K] (activations with `skip`,
 * weights with skip NULL): scale[r] = max |A[r,k]| over the kept columns (fp32);
 * q[r,k] = e4m3(fl32(A[r,k] * fl32(448 / scale[r]))); skipped columns and zero rows give
 * code 0. */
void oracle_absmax_quantize_rows_e4m3(const uint16_t *A, int64_t R, int64_t K,
                                      const uint8_t *skip, uint8_t *q, float *scale)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        const uint16_t *row = A + r * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (skip && skip[k])
                continue;
            float a = fabsf(oracle_half_to_float(row[k]));
            if (a > amax)
                amax = a;
        }
        scale[r] = amax;
        uint8_t *qr = q + r * K;
        if (amax == 0.0f) {
            for (int64_t k = 0; k < K; ++k)
                qr[k] = 0;
            continue;
        }
        float s = 448.0f / amax;
        for (int64_t k = 0; k < K; ++k) {
            if (skip && skip[k]) {
                qr[k] = 0;
                continue;
            }
            float v = oracle_half_to_float(row[k]) * s;
            qr[k] = oracle_e4m3_from_float(v);
        }
    }
}

/* The e4m3 product acc[i,n] = sum_k dec(A[rows[i],k]) * dec(B[n,k]) in fp64.  Every
 * product of two e4m3 values has at most 8 significant bits between 2^-18 and 2^17, so
 * sums of up to 2^16 of them are exact in fp64: acc is the exact product. */
void oracle_e4m3_matmul(const uint8_t *A, const uint8_t *B, int64_t nrows,
                        const int64_t *rows, int64_t N, int64_t K, double *acc)
{
    double dec[256];                 /* the 256 decoded values, from the decoder above */
    for (int c = 0; c < 256; ++c)
        dec[c] = oracle_e4m3_to_double((uint8_t)c);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t *a = A + (rows ? rows[i] : i) * K;
            const uint8_t *b = B + n * K;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += dec[a[k]] * dec[b[k]];
            acc[i * N + n] = s;
        }
    }
}

/* The whole e4m3 forward for a subset of rows, in fp64:
 *   C[i,n] = acc[i,n] * SCx[t] * SCB[n] / 448^2
 *          + sum_{j < n_o} X[t, idx[j]] * dec(CB[n, idx[j]]) * SCB[n] / 448 + bias[n]
 * with the mask and SCx over ALL rows of X, as in the int8 forward. */
int64_t oracle_linear_forward_rows_e4m3(const uint16_t *X, int64_t T, int64_t K,
                                        const uint8_t *CB, const float *SCB,
                                        const uint16_t *bias, int64_t N, float threshold,
                                        const int64_t *rows, int64_t nrows,
                                        uint32_t *mask_words, int32_t *idx, int32_t *n_o,
                                        uint8_t *Xq, float *SCx, double *acc, double *C)
{
    uint8_t *is_outlier = (uint8_t *)malloc((size_t)(K > 0 ? K : 1));
    if (!is_outlier)
        return -1;
    oracle_outlier_scan(X, T, K, threshold, is_outlier, mask_words, idx, n_o);
    oracle_absmax_quantize_rows_e4m3(X, T, K, is_outlier, Xq, SCx);
    oracle_e4m3_matmul(Xq, CB, nrows, rows, N, K, acc);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t t = rows ? rows[i] : i;
            double main_part = acc[i * N + n] * (double)SCx[t] * (double)SCB[n]
                               / (448.0 * 448.0);
            double out_part = 0.0;
            for (int32_t j = 0; j < *n_o; ++j) {
                int64_t k = idx[j];
                double w = oracle_e4m3_to_double(CB[n * K + k]) * (double)SCB[n] / 448.0;
                out_part += (double)oracle_half_to_float(X[t * K + k]) * w;
            }
            double b = bias ? (double)oracle_half_to_float(bias[n]) : 0.0;
            C[i * N + n] = main_part + out_part + b;
        }
    }
    free(is_outlier);
    return 0;
}

/* Backward of the fp16-weight training mode (the blog's "用法" names it for int8/fp16
 * mixed-precision training and gives no gradient formulas): the backward of
 * y = x W^T + b passed straight through the quantisation, in fp64 --
 *   dX[t,k] = sum_n dY[t,n] W[n,k],   dW[n,k] = sum_t dY[t,n] X[t,k],   db[n] = sum_t dY[t,n].
 * X [T,K], W [N,K], dY [T,N] fp16 (bits); outputs fp64, any of them NULL to skip. */
void oracle_linear_backward(const uint16_t *X, const uint16_t *W, const uint16_t *dY,
                            int64_t T, int64_t N, int64_t K, double *dX, double *dW,
                            double *db)
{
    if (dX) {
        #pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; ++t)
            for (int64_t k = 0; k < K; ++k) {
                double s = 0.0;
                for (int64_t n = 0; n < N; ++n)
                    s += (double)oracle_half_to_float(dY[t * N + n]) *
                         (double)oracle_half_to_float(W[n * K + k]);
                dX[t * K + k] = s;
            }
    }
    if (dW) {
        #pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t k = 0; k < K; ++k) {
                double s = 0.0;
                for (int64_t t = 0; t < T; ++t)
                    s += (double)oracle_half_to_float(dY[t * N + n]) *
                         (double)oracle_half_to_float(X[t * K + k]);
                dW[n * K + k] = s;
            }
    }
    if (db) {
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t t = 0; t < T; ++t)
                s += (double)oracle_half_to_float(dY[t * N + n]);
            db[n] = s;
        }
    }
}

/* The weight the int8 forward computes with ("用法": CB * SCB / 127 recovers it), in the
 * fp32 arithmetic the library's dequantisation states: W'[n,k] = fl32(CB[n,k] *
 * fl32(SCB[n] / 127)); with e4m3 codes (e4m3 != 0) their exact values times
 * fl32(SCB[n] / 448). */
void oracle_dequantize_weight(const uint8_t *CB, const float *SCB, int64_t N, int64_t K,
                              int32_t e4m3, float *W)
{
    for (int64_t n = 0; n < N; ++n) {
        const float s = SCB[n] / (e4m3 ? 448.0f : 127.0f);
        for (int64_t k = 0; k < K; ++k) {
            const float c = e4m3 ? (float)oracle_e4m3_to_double(CB[n * K + k])
                                 : (float)(int8_t)CB[n * K + k];
            W[n * K + k] = c * s;
        }
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
