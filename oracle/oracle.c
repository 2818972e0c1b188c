/*
 * oracle.c -- plain, slow, obviously correct CPU restatement of the LLM.int8() linear
 * layer, written from the pages' definitions.  TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * Pages followed:
 *   [P5] "PyTorch 2.9 支持 LLM.int8()：大模型低比特推理的工程突破" (yongjin360.com/news/208476)
 *        section "LLM.int8() 是怎么做到几乎无损的": item 1 per-channel weight quantization,
 *        item 2 dynamic activation quantization (round, clamp to [-127,127]),
 *        item 3 outlier columns kept in fp16, results merged;
 *        section "如何在 PyTorch 2.9 中启用 LLM.int8 推理": Linear8bitLt(has_fp16_weights=False).
 *   [P2] "8位量化实战：离群值处理与显存优化避坑指南" (zwxr.cn/news/257102)
 *        opening summary (vector-wise quantization + mixed-precision decomposition);
 *        section 2.3: Y = X_O . W_O (fp16) + quantize(X_R) . quantize(W_R) (int8),
 *        outlier column <=> column max |x| exceeds the threshold (default 6.0).
 *
 * Readings taken where the pages are silent or garbled:
 *   - one activation scale per ROW of X, taken over the regular columns only;
 *   - "round" is round-half-to-even (torch.round), done with nearbyint/nearbyintf under
 *     the default FE_TONEAREST mode;
 *   - scales are float32: s = absmax / 127.0f, q = round(x / s), both IEEE float divisions;
 *   - an all-zero row (or a row whose columns are all outliers) gets s = 0 and q = 0;
 *   - the outlier test is strict: |x| > threshold, compared in float32; a negative
 *     threshold is treated as 0, a NaN threshold is an error;
 *   - the outlier term uses W_hat = fp16(Wq * w_scale), since no fp16 weights are kept;
 *   - Y is the binary16 rounding of the double-precision sum A*sx*sw + P + bias.
 *
 * Parity pins: tests/test_oracle_pins.py (hand-worked examples, invariants, closed-form
 * special cases, exhaustive binary16 conversion against numpy, the error bound against
 * the unquantized product).
 */
#include "oracle.h"

#include <math.h>
#include <stddef.h>
#include <stdlib.h>

/* ------------------------------------------------------------------ binary16 */

double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exponent = (h >> 10) & 0x1f;
    int mantissa = h & 0x3ff;
    double v;
    if (exponent == 0) {
        v = ldexp((double)mantissa, -24);                 /* subnormal: m * 2^-24 */
    } else if (exponent == 31) {
        v = mantissa ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + mantissa), exponent - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

uint16_t oracle_half_from_double(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7e00;
    /* 65520 is halfway between the largest finite half (65504) and 2^16: ties go to the
     * even neighbour, which is the overflow to infinity. */
    if (a >= 65520.0) return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: integer multiple of 2^-24, rounded to nearest even */
        double q = nearbyint(a * ldexp(1.0, 24));
        return sign | (uint16_t)q;                       /* q == 1024 is the smallest normal */
    }
    int e2;
    double f = frexp(a, &e2);                            /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                                      /* a = (2f) * 2^e, 2f in [1, 2) */
    double scaled = nearbyint(2.0 * f * 1024.0);         /* in [1024, 2048] */
    if (scaled == 2048.0) {
        scaled = 1024.0;
        e += 1;
    }
    if (e + 15 >= 31) return sign | 0x7c00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)scaled - 1024));
}

static float half_to_float(uint16_t h) { return (float)oracle_half_to_double(h); }

/* round(v) to nearest, ties to even, then clamp to the symmetric int8 range */
static int8_t round_clamp_127(float v)
{
    float r = nearbyintf(v);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* ------------------------------------------------------------------ weights */

int oracle_quant_weight(const uint16_t *W, int64_t N, int64_t K, int8_t *Wq, float *w_scale)
{
    if (!W || !Wq || !w_scale || N <= 0 || K <= 0) return ORACLE_EINVAL;
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *w = W + n * K;
        float absmax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(half_to_float(w[k]));
            if (v > absmax) absmax = v;
        }
        float s = absmax / 127.0f;
        w_scale[n] = s;
        for (int64_t k = 0; k < K; ++k)
            Wq[n * K + k] = (absmax == 0.0f) ? 0 : round_clamp_127(half_to_float(w[k]) / s);
    }
    return 0;
}

/* ------------------------------------------------------------------ activations */

static float effective_threshold(float threshold) { return threshold < 0.0f ? 0.0f : threshold; }

int oracle_outlier_columns(const uint16_t *X, int64_t M, int64_t K, float threshold,
                           uint32_t *mask, int32_t *cols, int32_t *n_outliers)
{
    if (!X || !mask || !cols || !n_outliers || M <= 0 || K <= 0) return ORACLE_EINVAL;
    if (isnan(threshold)) return ORACLE_EINVAL;
    float t = effective_threshold(threshold);
    int64_t words = (K + 31) / 32;
    for (int64_t w = 0; w < words; ++w) mask[w] = 0;
    int32_t count = 0;
    for (int64_t j = 0; j < K; ++j) {
        int outlier = 0;
        for (int64_t i = 0; i < M; ++i)
            if (fabsf(half_to_float(X[i * K + j])) > t) outlier = 1;
        if (outlier) {
            mask[j / 32] |= (uint32_t)1 << (j % 32);
            cols[count++] = (int32_t)j;
        }
    }
    *n_outliers = count;
    return 0;
}

static int is_outlier(const uint32_t *mask, int64_t j) { return (mask[j / 32] >> (j % 32)) & 1; }

/* absmax of one row over the regular columns */
static float row_absmax(const uint16_t *x, int64_t K, const uint32_t *mask)
{
    float absmax = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
        if (is_outlier(mask, j)) continue;
        float v = fabsf(half_to_float(x[j]));
        if (v > absmax) absmax = v;
    }
    return absmax;
}

/* one row quantized with the absmax given: scale = absmax / 127, q = round(x / scale) */
static void quantize_with_absmax(const uint16_t *x, int64_t K, const uint32_t *mask,
                                 float absmax, int8_t *q, float *scale)
{
    float s = absmax / 127.0f;
    *scale = s;
    for (int64_t j = 0; j < K; ++j)
        q[j] = (is_outlier(mask, j) || absmax == 0.0f) ? 0 : round_clamp_127(half_to_float(x[j]) / s);
}

/* one row: absmax over the regular columns, scale, quantize */
static void quantize_one_row(const uint16_t *x, int64_t K, const uint32_t *mask,
                             int8_t *q, float *scale)
{
    quantize_with_absmax(x, K, mask, row_absmax(x, K, mask), q, scale);
}

/* [P5] section "LLM.int8() 是怎么做到几乎无损的", item 2, as its snippet is written: one
 * absmax for the whole activation tensor (over the regular columns, as for the rows). */
static float tensor_absmax(const uint16_t *X, int64_t M, int64_t K, const uint32_t *mask)
{
    float absmax = 0.0f;
    for (int64_t i = 0; i < M; ++i) {
        float a = row_absmax(X + i * K, K, mask);
        if (a > absmax) absmax = a;
    }
    return absmax;
}

int oracle_quantize_tensor(const uint16_t *X, int64_t M, int64_t K, const uint32_t *mask,
                           int8_t *Xq, float *row_scale)
{
    if (!X || !mask || !Xq || !row_scale || M <= 0 || K <= 0) return ORACLE_EINVAL;
    float absmax = tensor_absmax(X, M, K, mask);
    for (int64_t i = 0; i < M; ++i)
        quantize_with_absmax(X + i * K, K, mask, absmax, Xq + i * K, row_scale + i);
    return 0;
}

int oracle_quantize_rows(const uint16_t *X, int64_t M, int64_t K, const uint32_t *mask,
                         int8_t *Xq, float *row_scale)
{
    if (!X || !mask || !Xq || !row_scale || M <= 0 || K <= 0) return ORACLE_EINVAL;
    for (int64_t i = 0; i < M; ++i)
        quantize_one_row(X + i * K, K, mask, Xq + i * K, row_scale + i);
    return 0;
}

/* ------------------------------------------------------------------ products */

static int dot_i8(const int8_t *a, const int8_t *b, int64_t K, int32_t *out)
{
    int64_t acc = 0;
    for (int64_t k = 0; k < K; ++k) acc += (int64_t)a[k] * (int64_t)b[k];
    if (acc > INT32_MAX || acc < INT32_MIN) return ORACLE_ERANGE;
    *out = (int32_t)acc;
    return 0;
}

int oracle_gemm_i32(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                    int32_t *A)
{
    if (!Xq || !Wq || !A || M <= 0 || N <= 0 || K <= 0) return ORACLE_EINVAL;
    int status = 0;
    #pragma omp parallel for schedule(static) reduction(min:status)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t n = 0; n < N; ++n) {
            int rc = dot_i8(Xq + i * K, Wq + n * K, K, &A[i * N + n]);
            if (rc < status) status = rc;
        }
    return status;
}

int oracle_outlier_weights(const int8_t *Wq, const float *w_scale, int64_t N, int64_t K,
                           const int32_t *cols, int32_t n_out, uint16_t *W_hat)
{
    if (!Wq || !w_scale || N <= 0 || K <= 0 || n_out < 0 || n_out > K) return ORACLE_EINVAL;
    if (n_out > 0 && (!cols || !W_hat)) return ORACLE_EINVAL;
    for (int64_t n = 0; n < N; ++n)
        for (int32_t r = 0; r < n_out; ++r) {
            float w = (float)Wq[n * K + cols[r]] * w_scale[n];   /* float product, then fp16 */
            W_hat[n * n_out + r] = oracle_half_from_double((double)w);
        }
    return 0;
}

/* ------------------------------------------------------------------ the layer */

/* W16 (nullable): the layer's own fp16 weights [N, K]; when given, the outlier columns take
 * their weights from it instead of rebuilding them from the int8 weights. */
static int forward_rows(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                        const float *w_scale, const uint16_t *W16, const uint16_t *bias,
                        int64_t N, float threshold, int per_tensor, const int64_t *rows,
                        int64_t n_rows, uint16_t *Y_rows, int32_t *A_rows)
{
    if (!X || !Wq || !w_scale || !rows || !Y_rows || M <= 0 || N <= 0 || K <= 0 || n_rows < 0)
        return ORACLE_EINVAL;
    if (isnan(threshold)) return ORACLE_EINVAL;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= M) return ORACLE_EINVAL;

    int64_t words = (K + 31) / 32;
    uint32_t *mask = (uint32_t *)malloc((size_t)words * sizeof(uint32_t));
    int32_t *cols = (int32_t *)malloc((size_t)K * sizeof(int32_t));
    if (!mask || !cols) { free(mask); free(cols); return ORACLE_EINVAL; }
    int32_t n_out = 0;
    int status = oracle_outlier_columns(X, M, K, threshold, mask, cols, &n_out);

    uint16_t *W_hat = NULL;
    if (status == 0 && n_out > 0) {
        W_hat = (uint16_t *)malloc((size_t)N * (size_t)n_out * sizeof(uint16_t));
        if (!W_hat) status = ORACLE_EINVAL;
        else if (W16) {
            for (int64_t n = 0; n < N; ++n)
                for (int32_t o = 0; o < n_out; ++o) W_hat[n * n_out + o] = W16[n * K + cols[o]];
        } else status = oracle_outlier_weights(Wq, w_scale, N, K, cols, n_out, W_hat);
    }

    /* per-tensor scale: one absmax over every row of X, whichever rows are returned */
    float t_absmax = (status == 0 && per_tensor) ? tensor_absmax(X, M, K, mask) : 0.0f;
    if (status == 0) {
        #pragma omp parallel for schedule(dynamic, 1) reduction(min:status)
        for (int64_t r = 0; r < n_rows; ++r) {
            const uint16_t *x = X + rows[r] * K;
            int8_t *xq = (int8_t *)malloc((size_t)K);
            if (!xq) { status = ORACLE_EINVAL; continue; }
            float sx;
            if (per_tensor) quantize_with_absmax(x, K, mask, t_absmax, xq, &sx);
            else quantize_one_row(x, K, mask, xq, &sx);
            for (int64_t n = 0; n < N; ++n) {
                int32_t a;
                int rc = dot_i8(xq, Wq + n * K, K, &a);
                if (rc < status) status = rc;
                /* outlier term: fp16 operands, summed exactly enough in double */
                double p = 0.0;
                for (int32_t o = 0; o < n_out; ++o)
                    p += oracle_half_to_double(x[cols[o]]) *
                         oracle_half_to_double(W_hat[n * n_out + o]);
                double b = bias ? oracle_half_to_double(bias[n]) : 0.0;
                double y = (double)a * (double)sx * (double)w_scale[n] + p + b;
                Y_rows[r * N + n] = oracle_half_from_double(y);
                if (A_rows) A_rows[r * N + n] = a;
            }
            free(xq);
        }
    }
    free(W_hat);
    free(cols);
    free(mask);
    return status;
}

int oracle_linear_forward_rows(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                               const float *w_scale, const uint16_t *bias, int64_t N,
                               float threshold, const int64_t *rows, int64_t n_rows,
                               uint16_t *Y_rows, int32_t *A_rows)
{
    return forward_rows(X, M, K, Wq, w_scale, NULL, bias, N, threshold, 0, rows, n_rows,
                        Y_rows, A_rows);
}

int oracle_linear_forward_rows_ex(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                                  const float *w_scale, const uint16_t *W16,
                                  const uint16_t *bias, int64_t N, float threshold,
                                  int per_tensor, const int64_t *rows, int64_t n_rows,
                                  uint16_t *Y_rows, int32_t *A_rows)
{
    return forward_rows(X, M, K, Wq, w_scale, W16, bias, N, threshold, per_tensor != 0, rows,
                        n_rows, Y_rows, A_rows);
}

int oracle_linear_forward_rows_w16(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                                   const float *w_scale, const uint16_t *W16,
                                   const uint16_t *bias, int64_t N, float threshold,
                                   const int64_t *rows, int64_t n_rows, uint16_t *Y_rows,
                                   int32_t *A_rows)
{
    if (!W16) return ORACLE_EINVAL;
    return forward_rows(X, M, K, Wq, w_scale, W16, bias, N, threshold, 0, rows, n_rows, Y_rows,
                        A_rows);
}

int oracle_linear_forward(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                          const float *w_scale, const uint16_t *bias, int64_t N,
                          float threshold, uint16_t *Y)
{
    if (M <= 0) return ORACLE_EINVAL;
    int64_t *rows = (int64_t *)malloc((size_t)M * sizeof(int64_t));
    if (!rows) return ORACLE_EINVAL;
    for (int64_t i = 0; i < M; ++i) rows[i] = i;
    int status = oracle_linear_forward_rows(X, M, K, Wq, w_scale, bias, N, threshold, rows, M,
                                            Y, NULL);
    free(rows);
    return status;
}

/* ------------------------------------------------------------------ activation statistics */

static int cmp_float(const void *a, const void *b)
{
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

/* [P2] section 5.1 (statistics before choosing a threshold): the largest |x|, the 0.99
 * quantile of |x| over every element (order statistics of the sorted values, linear
 * interpolation between the two around position 0.99 (n - 1)), their ratio
 * max / (q99 + 1e-6), and the absmax of every column.  out: {max, q99, ratio}. */
int oracle_activation_stats(const uint16_t *X, int64_t M, int64_t K, float *col_absmax,
                            double *out)
{
    if (!X || !out || M <= 0 || K <= 0) return ORACLE_EINVAL;
    int64_t n = M * K;
    float *v = (float *)malloc((size_t)n * sizeof(float));
    if (!v) return ORACLE_EINVAL;
    float mx = 0.0f;
    for (int64_t j = 0; j < K && col_absmax; ++j) col_absmax[j] = 0.0f;
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < K; ++j) {
            float a = fabsf(half_to_float(X[i * K + j]));
            v[i * K + j] = a;
            if (a > mx) mx = a;
            if (col_absmax && a > col_absmax[j]) col_absmax[j] = a;
        }
    qsort(v, (size_t)n, sizeof(float), cmp_float);
    double pos = 0.99 * (double)(n - 1);
    int64_t lo = (int64_t)floor(pos);
    double frac = pos - (double)lo;
    double a = v[lo], b = lo + 1 < n ? v[lo + 1] : v[lo];
    double q99 = a + frac * (b - a);
    out[0] = mx;
    out[1] = q99;
    out[2] = (double)mx / (q99 + 1e-6);
    free(v);
    return 0;
}
