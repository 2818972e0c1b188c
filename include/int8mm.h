/*
 * int8mm.h -- C ABI of the B200 (sm_100a) LLM.int8() linear layer, libint8mm.so.
 *
 * The layer (Y = X . W^T with vector-wise int8 quantization and mixed-precision
 * decomposition) is defined on two pages, cited below by title and section:
 *   [P5] "PyTorch 2.9 支持 LLM.int8()：大模型低比特推理的工程突破" (yongjin360.com/news/208476)
 *   [P2] "8位量化实战：离群值处理与显存优化避坑指南" (zwxr.cn/news/257102)
 *
 * Conventions for every entry point:
 *   - Matrices are row-major with K (the input-feature axis) contiguous.
 *   - Half-precision data is IEEE binary16 (passed as void*; the ABI has no half type).
 *   - Every pointer is a caller-owned DEVICE pointer on the current CUDA device, unless
 *     stated otherwise; the library allocates nothing and keeps no state between calls
 *     (except the static scratch of int8_linear_forward_noalloc, described there).
 *     Matrix and vector pointers must be 16-byte aligned.
 *   - K must be a multiple of 16 (each row must start on a 16-byte boundary for the
 *     tensor-memory-access unit); 1 <= M, N and K <= INT8MM_MAX_K.
 *   - Work is enqueued on `stream` (NULL = the legacy default stream) and the call
 *     returns without waiting; the return value reports argument and launch errors only.
 *     Kernel-side failures (a bounded wait that gave up) are written as a negative code
 *     to a device status word and read with int8_read_device_status().
 *   - Results are deterministic: the same inputs give the same bits on every call.
 *   - The forward's kernels are launched with programmatic dependent launch: a kernel may
 *     start while the kernel before it on the stream is finishing, and it waits for that
 *     kernel before it reads X (or any activation data) and before it writes anything.  One
 *     read comes before that wait: with M <= 8 (the one-launch decode route) each CTA starts
 *     copying its rows of Wq at once.  So Wq must not be written by the kernel launched just
 *     before the forward on the same stream.  Weights made by int8_quant_weight on the same
 *     stream are safe to use at once: its kernel never lets the next launch start early.
 */
#ifndef INT8MM_H
#define INT8MM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *int8mm_stream_t; /* the same type as cudaStream_t */

#define INT8MM_MAX_K 65536

/* status codes */
#define INT8MM_OK 0
#define INT8MM_ERR_NULL (-1)         /* a required pointer is NULL */
#define INT8MM_ERR_SHAPE (-2)        /* M, N or K out of range */
#define INT8MM_ERR_ALIGN (-3)        /* K % 16 != 0, or a pointer not 16-byte aligned */
#define INT8MM_ERR_THRESHOLD (-4)    /* threshold is NaN */
#define INT8MM_ERR_WORKSPACE (-5)    /* workspace NULL, misaligned or too small */
#define INT8MM_ERR_CUDA (-6)         /* a CUDA runtime or launch error */
#define INT8MM_ERR_DEVICE (-7)       /* the current device is not sm_100 */
#define INT8MM_ERR_TIMEOUT (-8)      /* device side: a bounded wait gave up */
#define INT8MM_ERR_OVERFLOW (-9)     /* device side: an outlier count beyond K */
#define INT8MM_ERR_SCRATCH (-10)     /* shape beyond int8_linear_forward_noalloc's scratch */
#define INT8MM_ERR_FLAGS (-11)       /* unknown bits in the flags of int8_linear_forward_ex */

/* flags of int8_linear_forward_ex */
#define INT8MM_PER_TENSOR_SCALE 1u   /* one activation scale for the whole of X */
#define INT8MM_PAIR_TILES 2u         /* M > 128: 256 x 256 product tiles on CTA pairs */

/* Bytes of the static device scratch behind int8_linear_forward_noalloc (per device). */
#define INT8MM_NOALLOC_SCRATCH_BYTES (512 * 1024)

/* Human-readable name of a status code (static string, never NULL). */
const char *int8_status_string(int status);

/*
 * Per-output-channel weight quantization, done once when the layer is loaded.
 * [P5] section "LLM.int8() 是怎么做到几乎无损的", item 1:
 *   w_scale[n] = max_k |W[n,k]| / 127;  Wq[n,k] = round(W[n,k] / w_scale[n]).
 * The scale is a float32 IEEE division; round is to nearest, ties to even; the result is
 * clamped to [-127, 127]; an all-zero channel gets scale 0 and all-zero codes.
 *   W        [in]  binary16 [N, K]
 *   Wq       [out] int8     [N, K]
 *   w_scale  [out] float32  [N]
 */
int int8_quant_weight(const void *W, int N, int K, int8_t *Wq, float *w_scale,
                      int8mm_stream_t stream);

/*
 * Bytes of device workspace int8_linear_forward and int8_quantize_rows need for an
 * [M, K] x [N, K]^T layer.  The workspace holds the device status word (its first int32),
 * the outlier-column mask and list, the row scales, the int8 activations and the fp16
 * outlier operands, sized for the worst case (every column an outlier).  Zero it once
 * before first use (kernels only ever write a nonzero code into the status word).
 * Returns 0 for out-of-range sizes.
 */
size_t int8_linear_workspace_size(int M, int N, int K);

/*
 * The LLM.int8() linear layer, [P2] section 2.3 with [P5] items 1-3:
 *   O   = { j : max_i |X[i,j]| > threshold }          (outlier feature columns)
 *   sx  = per row i, max over j not in O of |X[i,j]|, divided by 127 (float32)
 *   Xq  = round(X / sx) on the regular columns, 0 on O   (X / sx the float32 IEEE quotient,
 *         rounded to nearest, ties to even; [-127,127])
 *   Y   = fp16( (Xq . Wq^T)[i,n] * sx[i] * w_scale[n]         (int8 x int8 -> int32)
 *               + sum_{j in O} X[i,j] * W_hat[n,j]             (fp16 operands, fp32 sum)
 *               + bias[n] )
 * with W_hat = fp16(Wq * w_scale): the layer keeps no fp16 weights ([P5] section
 * "如何在 PyTorch 2.9 中启用 LLM.int8 推理", has_fp16_weights=False).
 *   X          [in]  binary16 [M, K]
 *   Wq, w_scale[in]  from int8_quant_weight, int8 [N, K] and float32 [N]
 *   bias       [in]  binary16 [N], or NULL for none
 *   threshold  [in]  outlier threshold (the pages' default is 6.0); a negative value acts
 *                    as 0 (every column holding a nonzero value is an outlier); +inf turns
 *                    the fp16 term off; NaN is rejected
 *   Y          [out] binary16 [M, N]
 *   workspace  [in/out] ws_bytes >= int8_linear_workspace_size(M, N, K), 256-byte aligned
 * Calls that share a workspace must not overlap on the GPU.
 */
int int8_linear_forward(const void *X, int M, int K, const int8_t *Wq, const float *w_scale,
                        const void *bias, int N, float threshold, void *Y, void *workspace,
                        size_t ws_bytes, int8mm_stream_t stream);

/*
 * The layer that keeps its fp16 weights ([P5] section "如何在 PyTorch 2.9 中启用 LLM.int8
 * 推理", has_fp16_weights=True): as int8_linear_forward, except that the outlier term reads
 * the layer's own fp16 weights, sum_{j in O} X[i,j] * W16[n,j], in place of the rebuilt
 * W_hat = fp16(Wq * w_scale).  The int8 term is unchanged (Wq and w_scale still come from
 * int8_quant_weight of the same weights).
 *   W16        [in]  binary16 [N, K], row-major, 16-byte aligned, read only at the outlier
 *                    columns; NULL is rejected (INT8MM_ERR_NULL)
 * Every other argument, the workspace and the error codes are as for int8_linear_forward.
 */
int int8_linear_forward_fp16w(const void *X, int M, int K, const int8_t *Wq,
                              const float *w_scale, const void *W16, const void *bias, int N,
                              float threshold, void *Y, void *workspace, size_t ws_bytes,
                              int8mm_stream_t stream);

/*
 * int8_linear_forward with every option of the layer:
 *   W16    [in]  NULL, or the layer's fp16 weights as for int8_linear_forward_fp16w
 *   flags  [in]  0, or INT8MM_PER_TENSOR_SCALE: one activation scale for the whole of X,
 *                sx = (max over every row i and regular column j of |X[i,j]|) / 127, every
 *                row quantized with it ([P5] section "LLM.int8() 是怎么做到几乎无损的", item 2,
 *                as its snippet is written; the default one-per-row scale follows the
 *                vector-wise reading of [P2]);
 *                INT8MM_PAIR_TILES: for M > 128, compute the products in 256 x 256 tiles, each
 *                shared by a pair of CTAs (tcgen05 cta_group::2: each CTA loads half of the
 *                operands), instead of 128 x 256 tiles on single CTAs.  Same results, bit for
 *                bit in the integer stages; it moves a third less operand data per multiply-add
 *                but, measured under the 1 kW power cap, is not faster (the default is the
 *                single-CTA tile).  Other bits: INT8MM_ERR_FLAGS.
 *   acc    [out] NULL, or int32 [M, N]: the int8 accumulators, as int8_linear_forward_acc
 * Every other argument, the workspace and the error codes are as for int8_linear_forward.
 */
int int8_linear_forward_ex(const void *X, int M, int K, const int8_t *Wq, const float *w_scale,
                           const void *W16, const void *bias, int N, float threshold,
                           unsigned flags, void *Y, int32_t *acc, void *workspace,
                           size_t ws_bytes, int8mm_stream_t stream);

/*
 * Statistics of the layer's input for choosing the threshold ([P2] section 5.1, which
 * compares the largest |x| with its 0.99 quantile: a ratio far above 1 flags outliers), over
 * every element of X:
 *   out        [out] double [3] (device): max |X|; q99 = the 0.99 quantile of |X| (the sorted
 *                    values interpolated linearly at position 0.99 (M K - 1)); max / (q99 + 1e-6)
 *   col_absmax [out] float32 [K], or NULL: max_i |X[i,j]| of each column (a column is an
 *                    outlier when this exceeds the threshold)
 *   workspace  [scratch] ws_bytes >= int8_activation_stats_workspace_size(), 256-byte aligned
 * M K must be below 2^32.  NaN or infinite inputs give unspecified statistics.
 */
size_t int8_activation_stats_workspace_size(void);
int int8_activation_stats(const void *X, int M, int K, float *col_absmax, double *out,
                          void *workspace, size_t ws_bytes, int8mm_stream_t stream);

/*
 * The outlier test of [P2] section 2.3 applied to column maxima gathered elsewhere, for a
 * layer whose tokens are split across GPUs: every rank takes the column absmax of its own rows
 * (int8_activation_stats), a MAX all-reduce makes them the maxima over all rows, and this call
 * turns them into one extra activation row,
 *   row[j] = binary16(col_absmax[j])  if col_absmax[j] > threshold,  0 otherwise,
 * which the rank appends to its rows before int8_linear_forward.  That row exceeds the
 * threshold in exactly the global outlier columns (the maxima are binary16 magnitudes, so the
 * conversion is exact) and no real row's scale or codes change; its output row is dropped.
 *   col_absmax [in]  float32 [K]
 *   threshold  [in]  as for int8_linear_forward (negative acts as 0, +inf marks nothing,
 *                    NaN is rejected)
 *   row        [out] binary16 [K]
 */
int int8_outlier_row(const float *col_absmax, int K, float threshold, void *row,
                     int8mm_stream_t stream);

/*
 * The two halves of int8_linear_forward, for callers that time or schedule them apart:
 * int8_linear_forward is exactly int8_linear_quantize followed by int8_linear_matmul with
 * the same arguments, workspace and stream.  Arguments are as for int8_linear_forward.
 *
 * int8_linear_quantize: the activation side.  For M > 16: outlier columns, per-row scales,
 *   int8 activations and the compacted fp16 outlier operands (activations and
 *   W_hat = fp16(Wq * w_scale)), written into the workspace.  For few tokens (the
 *   weight-streaming regime): with M <= 8, K % 128 == 0 and K <= 8192 it enqueues nothing (one
 *   kernel in int8_linear_matmul does the whole layer); with M <= 16 otherwise under the same
 *   K limits it enqueues one kernel that quantizes the activations once into the workspace;
 *   for longer rows with M <= 16 it enqueues nothing (one kernel quantizes next to the tensor
 *   cores).
 * int8_linear_matmul: the rest -- the int8 and fp16 products and the fused epilogue --
 *   reading what int8_linear_quantize left in the workspace.
 */
int int8_linear_quantize(const void *X, int M, int K, const int8_t *Wq, const float *w_scale,
                         int N, float threshold, void *workspace, size_t ws_bytes,
                         int8mm_stream_t stream);
int int8_linear_matmul(const void *X, int M, int K, const int8_t *Wq, const float *w_scale,
                       const void *bias, int N, float threshold, void *Y, void *workspace,
                       size_t ws_bytes, int8mm_stream_t stream);

/*
 * Diagnostic: int8_linear_forward that also writes the int32 accumulators
 * acc[i,n] = sum_k Xq[i,k] * Wq[n,k] (the int8 product of [P2] section 2.3 before
 * dequantization), int32 [M, N], 16-byte aligned.  Y is as for int8_linear_forward.
 */
int int8_linear_forward_acc(const void *X, int M, int K, const int8_t *Wq,
                            const float *w_scale, const void *bias, int N, float threshold,
                            void *Y, int32_t *acc, void *workspace, size_t ws_bytes,
                            int8mm_stream_t stream);

/*
 * Diagnostic: the quantization half of the layer alone (outlier detection and per-row
 * activation quantization, [P2] section 2.3 and [P5] item 2, as in int8_linear_forward).
 *   X            [in]  binary16 [M, K]
 *   Xq           [out] int8     [M, K] (0 in outlier columns)
 *   row_scale    [out] float32  [M]
 *   outlier_cols [out] int32    [K]: the outlier columns in ascending order, first
 *                      *n_outliers entries valid
 *   n_outliers   [out] int32    [1] (device memory)
 *   workspace    as for int8_linear_forward with N = 1
 */
int int8_quantize_rows(const void *X, int M, int K, float threshold, int8_t *Xq,
                       float *row_scale, int32_t *outlier_cols, int32_t *n_outliers,
                       void *workspace, size_t ws_bytes, int8mm_stream_t stream);

/*
 * Diagnostic: the int8 product alone, C[i,n] = sum_k Xq[i,k] * Wq[n,k], exact int32
 * (the int8 matrix multiplication of [P2] section 2.3, run on the tensor cores).
 *   Xq [in] int8 [M, K];  Wq [in] int8 [N, K];  C [out] int32 [M, N]
 *   dev_status [in/out] one int32 of device memory that receives a negative code if a
 *              bounded wait gives up (zero it before the first call)
 */
int int8_gemm_i32(const int8_t *Xq, const int8_t *Wq, int M, int N, int K, int32_t *C,
                  int32_t *dev_status, int8mm_stream_t stream);

/*
 * Diagnostic: the fp16 outlier weights alone,
 *   W_hat[n, r] = fp16(float(Wq[n, cols[r]]) * w_scale[n])   for r < *n_outliers
 * (the layer keeps no fp16 weights: [P5] section "如何在 PyTorch 2.9 中启用 LLM.int8 推理",
 * has_fp16_weights=False).  The product is rounded to float32, then to binary16 (ties to
 * even).
 *   outlier_cols, n_outliers [in] device int32, as written by int8_quantize_rows
 *   W_hat [out] binary16 [N, K] with row stride K; entries r >= *n_outliers are untouched
 */
int int8_outlier_weights(const int8_t *Wq, const float *w_scale, int N, int K,
                         const int32_t *outlier_cols, const int32_t *n_outliers, void *W_hat,
                         int8mm_stream_t stream);

/*
 * Diagnostic: int8_linear_forward_ex that also hands back what the forward's own kernels
 * computed on the way to Y, so that every intermediate of the method can be compared with
 * its definition: the outlier columns ([P2] section 2.3), the per-row (or per-tensor)
 * activation scales and codes ([P5] section "LLM.int8() 是怎么做到几乎无损的", item 2) and
 * the fp16 weights the outlier term multiplied ([P5] section "如何在 PyTorch 2.9 中启用
 * LLM.int8 推理", has_fp16_weights).  The values come from the kernels that produce Y for
 * this shape (the one-launch decode kernel, the few-token pair, the cluster kernel or the
 * tiled passes), not from a separate computation.  Every output pointer may be NULL.
 *   Xq           [out] int8 [M, K]: the codes, 0 in outlier columns
 *   row_scale    [out] float32 [M]: the activation scale of each row
 *   outlier_cols [out] int32 [K]: the outlier columns in ascending order, first *n_outliers
 *                      entries valid
 *   n_outliers   [out] int32 [1]
 *   W_hat        [out] binary16 [N, K]: at every outlier column j, W_hat[n, j] is the weight
 *                      the outlier term used (fp16(Wq[n,j] * w_scale[n]), or W16[n,j] when
 *                      W16 is given); entries of the other columns are left untouched
 * Every other argument, the workspace and the error codes are as for int8_linear_forward_ex;
 * Y and acc get the same bits as from int8_linear_forward_ex.  Output pointers must be
 * 16-byte aligned.  The extra writes make this call slower than the forward: it is meant for
 * tests and debugging, not for the hot path.
 */
int int8_linear_forward_trace(const void *X, int M, int K, const int8_t *Wq,
                              const float *w_scale, const void *W16, const void *bias, int N,
                              float threshold, unsigned flags, void *Y, int32_t *acc, int8_t *Xq,
                              float *row_scale, int32_t *outlier_cols, int32_t *n_outliers,
                              void *W_hat, void *workspace, size_t ws_bytes,
                              int8mm_stream_t stream);

/*
 * int8_linear_forward without a workspace argument, for few-token (decode) shapes.
 * The pages have no counterpart: this is a calling convention, not part of the method.
 * It serves callers that cannot allocate device memory where they call the layer -- a
 * stream being captured into a graph, an allocator that must not grow mid-step, or a C
 * host that has no way to hand over a workspace -- so it allocates nothing and calls no
 * allocating routine.  Its scratch (outlier list, int8 and outlier activations, row
 * scales) is a static device array of INT8MM_NOALLOC_SCRATCH_BYTES that every GPU which
 * loads the library holds until the process exits.
 *   X, Wq, w_scale, bias, threshold, Y   as for int8_linear_forward (same kernels, same bits)
 *   dev_status [in/out] one int32 of device memory that receives a negative code if a
 *              bounded device-side wait gives up (zero it first), or NULL to not be told
 * Limits: M <= 16, and a shape the few-token kernels take (K <= 8192 with K % 128 == 0, or
 * the single-kernel cluster path); anything else returns INT8MM_ERR_SCRATCH at once.
 * The first call on each device looks up that device's copy of the array (with the device
 * current); make that first call before any stream capture begins.
 * Every call on a device shares the one array and leaves its contents behind (nothing in
 * it needs to start at zero), so calls that overlap on the GPU -- on two streams, or from
 * two threads -- race and give wrong results; order them on one stream.
 */
int int8_linear_forward_noalloc(const void *X, int M, int K, const int8_t *Wq,
                                const float *w_scale, const void *bias, int N, float threshold,
                                void *Y, int32_t *dev_status, int8mm_stream_t stream);

/*
 * Waits for `stream`, then returns the device status word at dev_status (for the forward
 * and int8_quantize_rows, the word is the first int32 of the workspace): 0, or the
 * negative code a kernel wrote.  Returns INT8MM_ERR_CUDA if the stream itself failed.
 */
int int8_read_device_status(const int32_t *dev_status, int8mm_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
