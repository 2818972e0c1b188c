/*
 * oracle.h -- plain CPU reference of the LLM.int8() linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path includes, links or
 * loads this.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
 * and reference legs may call it.  It shares no code, header, table or helper
 * with the CUDA library under int8_mixed_precision_absmax_b200/csrc.
 *
 * Half-precision values are passed as their IEEE-754 binary16 bit patterns
 * (uint16_t); C99 has no half type.  All matrices are row-major, contiguous.
 * Every function returns 0 on success and a negative value on a bad argument.
 *
 * Pages followed (cited by title and section):
 *   [P5] "PyTorch 2.9 支持 LLM.int8()：大模型低比特推理的工程突破"
 *        (yongjin360.com/news/208476)
 *   [P2] "8位量化实战：离群值处理与显存优化避坑指南" (zwxr.cn/news/257102)
 */
#ifndef INT8_ABSMAX_ORACLE_H
#define INT8_ABSMAX_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_EINVAL (-22)
#define ORACLE_ERANGE (-34)

/* binary16 <-> double.  Decoding is exact; encoding rounds to nearest, ties to even. */
double   oracle_half_to_double(uint16_t h);
uint16_t oracle_half_from_double(double x);

/* [P5] section "LLM.int8() 是怎么做到几乎无损的", item 1 (per-output-channel weight
 * quantization): w_scale[n] = max_k |W[n,k]| / 127, Wq[n,k] = round(W[n,k] / w_scale[n]).
 * W: binary16 [N,K]; Wq: int8 [N,K]; w_scale: float [N]. */
int oracle_quant_weight(const uint16_t *W, int64_t N, int64_t K, int8_t *Wq, float *w_scale);

/* [P2] section 2.3 (the outlier-column split): column j is an outlier when some |X[i,j]|
 * exceeds the threshold.  mask: uint32 [ceil(K/32)] (bit j%32 of word j/32); cols: int32 [K]
 * ascending (the first *n_outliers entries are valid). */
int oracle_outlier_columns(const uint16_t *X, int64_t M, int64_t K, float threshold,
                           uint32_t *mask, int32_t *cols, int32_t *n_outliers);

/* [P5] item 2 (dynamic activation quantization), applied per row of X and only over the
 * regular (non-outlier) columns, per the quantize(X_R) term of [P2] section 2.3.
 * Xq: int8 [M,K] (0 in outlier columns); row_scale: float [M]. */
int oracle_quantize_rows(const uint16_t *X, int64_t M, int64_t K, const uint32_t *mask,
                         int8_t *Xq, float *row_scale);

/* int8 x int8 product A[i,n] = sum_k Xq[i,k] * Wq[n,k], accumulated in int64 and checked
 * to fit int32 (ORACLE_ERANGE otherwise). */
int oracle_gemm_i32(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                    int32_t *A);

/* The fp16 weights of the outlier columns, rebuilt from the int8 weights because the
 * layer keeps no fp16 copy ([P5] section "如何在 PyTorch 2.9 中启用 LLM.int8 推理",
 * has_fp16_weights=False): W_hat[n,r] = fp16(float(Wq[n,cols[r]]) * w_scale[n]).
 * W_hat: binary16 [N, n_out]. */
int oracle_outlier_weights(const int8_t *Wq, const float *w_scale, int64_t N, int64_t K,
                           const int32_t *cols, int32_t n_out, uint16_t *W_hat);

/* The whole layer, [P2] section 2.3:
 *   Y = X_O . W_hat_O^T (fp16 operands) + dequant(quantize(X_R) . quantize(W_R)^T) + bias.
 * bias may be NULL.  Y: binary16 [M,N]. */
int oracle_linear_forward(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                          const float *w_scale, const uint16_t *bias, int64_t N,
                          float threshold, uint16_t *Y);

/* The same layer evaluated only on the listed rows of X (the outlier set is still found
 * over all M rows).  Y_rows: binary16 [n_rows, N]; A_rows (nullable): int32 [n_rows, N].
 * Used to sample layers too large to evaluate whole on a CPU. */
int oracle_linear_forward_rows(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                               const float *w_scale, const uint16_t *bias, int64_t N,
                               float threshold, const int64_t *rows, int64_t n_rows,
                               uint16_t *Y_rows, int32_t *A_rows);

/* The layer that keeps its fp16 weights ([P5] section "如何在 PyTorch 2.9 中启用 LLM.int8
 * 推理": has_fp16_weights=True): as oracle_linear_forward_rows, except that the fp16 term uses
 * the kept weights of the outlier columns, W_hat[n,j] = W16[n,j], instead of rebuilding them
 * from Wq.  W16: binary16 [N, K], the weights Wq and w_scale were quantized from. */
int oracle_linear_forward_rows_w16(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                                   const float *w_scale, const uint16_t *W16,
                                   const uint16_t *bias, int64_t N, float threshold,
                                   const int64_t *rows, int64_t n_rows, uint16_t *Y_rows,
                                   int32_t *A_rows);

/* [P5] section "LLM.int8() 是怎么做到几乎无损的", item 2, with its snippet's granularity: one
 * scale for the whole activation tensor, absmax over every row and the regular columns,
 * divided by 127; each row quantized with it as oracle_quantize_rows does.  row_scale[i] holds
 * that one scale for every row. */
int oracle_quantize_tensor(const uint16_t *X, int64_t M, int64_t K, const uint32_t *mask,
                           int8_t *Xq, float *row_scale);

/* The layer with both options: W16 (nullable) as in oracle_linear_forward_rows_w16, and
 * per_tensor != 0 for one activation scale over the whole of X (oracle_quantize_tensor). */
int oracle_linear_forward_rows_ex(const uint16_t *X, int64_t M, int64_t K, const int8_t *Wq,
                                  const float *w_scale, const uint16_t *W16,
                                  const uint16_t *bias, int64_t N, float threshold,
                                  int per_tensor, const int64_t *rows, int64_t n_rows,
                                  uint16_t *Y_rows, int32_t *A_rows);

/* [P2] section 5.1: statistics of |X| for choosing a threshold.  col_absmax: float [K]
 * (nullable), the largest |X[i,j]| of each column; out: double [3] = {max |X|, the 0.99
 * quantile of |X| over all M K values (linear interpolation at position 0.99 (M K - 1) of the
 * sorted values), max / (q99 + 1e-6)}. */
int oracle_activation_stats(const uint16_t *X, int64_t M, int64_t K, float *col_absmax,
                            double *out);

#ifdef __cplusplus
}
#endif
#endif
