// kernels.cuh -- internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "int8mm.h"

namespace i8mm {

// ---------------------------------------------------------------- workspace layout
//
// One contiguous device buffer, every region 256-byte aligned:
//   header   int32[64]      [0] status word, [1] outlier count
//   mask     uint32[ceil(K/32)]    bit j%32 of word j/32 set <=> column j is an outlier
//   cols     int32[K]       outlier columns, ascending
//   xscale   float[M]       per-row activation scale
//   xq       int8[M*K]      quantized activations (0 in outlier columns)
//   xo       half[M*ldo]    outlier activations, compacted, zero-padded to a multiple of 64
//   wo       half[N*ldo]    outlier weights fp16(Wq*w_scale), compacted, zero-padded
// ldo = K rounded up to 64 (the fp16 operand tiles are 64 elements deep).
// The few-token path (M <= kSmallMP) adds: int8 activations padded to 16 rows and to a
// multiple of 256 columns (few_xq, int8[16*kpad]), the fp16 values of the outlier columns
// (few_xo, half[K*16], outlier r at [r*16 + i]) and the 16 row scales (few_sx); the outlier
// count and list use header[1] and cols.
constexpr int kSmallMP = 16;             // tokens per MMA (N of the swapped product)
constexpr int kSmallBN = 128;            // output channels per tile (M of the MMA)
constexpr int kSmallMaxSplits = 8;       // CTAs per cluster (portable cluster size)
constexpr int kSmallMaxKbPerSplit = 16;  // 128-byte k-blocks of X / Xq one CTA keeps in smem

struct WorkspaceLayout {
  size_t header, mask, wmax, cols, xscale, xq, xo, wo, few_xq, few_xo, few_sx, total;
  int ldo;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline WorkspaceLayout workspace_layout(int M, int N, int K) {
  WorkspaceLayout L;
  L.ldo = (K + 63) / 64 * 64;
  size_t off = 0;
  L.header = off; off = align256(off + 64 * sizeof(int32_t));
  L.mask = off;   off = align256(off + static_cast<size_t>((K + 31) / 32) * sizeof(uint32_t));
  L.wmax = off;   off = align256(off + static_cast<size_t>((K + 31) / 32) * sizeof(float));
  L.cols = off;   off = align256(off + static_cast<size_t>(K) * sizeof(int32_t));
  L.xscale = off; off = align256(off + static_cast<size_t>(M) * sizeof(float));
  L.xq = off;     off = align256(off + static_cast<size_t>(M) * K);
  L.xo = off;     off = align256(off + static_cast<size_t>(M) * L.ldo * sizeof(__half));
  L.wo = off;     off = align256(off + static_cast<size_t>(N) * L.ldo * sizeof(__half));
  L.few_xq = L.few_xo = L.few_sx = off;
  if (M <= kSmallMP) {
    const size_t kpad = static_cast<size_t>((K + 255) / 256) * 256;
    L.few_xq = off; off = align256(off + kSmallMP * kpad);
    L.few_xo = off; off = align256(off + static_cast<size_t>(K) * kSmallMP * sizeof(__half));
    L.few_sx = off; off = align256(off + kSmallMP * sizeof(float));
  }
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- launches
// Each returns cudaSuccess or the launch error; `pdl` lets the launch start while the
// previous kernel on the stream drains (the kernel waits on griddepcontrol before
// touching its inputs).

cudaError_t launch_quant_weight(const __half* W, int N, int K, int8_t* Wq, float* w_scale,
                                cudaStream_t stream);

// word_max (nullable): per 32-column word of the mask, the largest |x| over the word's regular
// columns and every row (the per-tensor activation scale is the largest of them / 127)
cudaError_t launch_colmask(const __half* X, int M, int K, float threshold, uint32_t* mask,
                           float* word_max, cudaStream_t stream, bool pdl);

cudaError_t launch_outlier_weights(const int8_t* Wq, const float* w_scale, int N, int K,
                                   const int32_t* cols, const int32_t* n_out, __half* W_hat,
                                   cudaStream_t stream);

struct RowQuantArgs {
  const __half* X;
  int M, K;
  const uint32_t* mask;
  int8_t* xq;
  float* xscale;
  __half* xo;           // nullable: skip the outlier-activation gather
  int ldo;
  int32_t* cols;        // written by block 0
  int32_t* n_out;       // written by block 0
  // outlier-weight gather (extra blocks after the M row blocks); wo nullable
  const int8_t* Wq;
  const float* w_scale;
  const __half* W16;    // nullable: the layer's fp16 weights [N, K] for the outlier columns
  __half* wo;
  int N;
  const float* word_max;  // nullable: one activation scale for all rows from colmask's maxima
  int32_t* status;
};
cudaError_t launch_rowquant(const RowQuantArgs& a, cudaStream_t stream, bool pdl);

// What a forward's own kernels computed on the way to Y, for the diagnostic
// int8_linear_forward_trace (every pointer nullable; all null on the normal path):
//   xq     int8 [M, K]  the activation codes (0 in outlier columns)
//   sx     f32 [M]      the row scales
//   flags  u8 [K / 8]   outlier bits, one byte per 8 columns (byte c bit e: column 8 c + e),
//                       the same bytes as the little-endian words of the workspace mask
//   what   half [N, K]  at each outlier column j, the fp16 weight the outlier term used
struct TraceSink {
  int8_t* xq = nullptr;
  float* sx = nullptr;
  uint8_t* flags = nullptr;
  __half* what = nullptr;
};

// trace.cu: the outlier list from outlier bits (bits of columns >= K ignored; cols and n_out
// nullable), and the tiled path's compacted outlier weights scattered to their columns.
cudaError_t launch_trace_cols(const uint32_t* mask, int K, int32_t* cols, int32_t* n_out,
                              cudaStream_t stream);
cudaError_t launch_trace_what(const __half* wo, int ldo, const int32_t* cols,
                              const int32_t* n_out, int N, int K, __half* W_hat,
                              cudaStream_t stream);

struct SmallArgs {
  const __half* X;
  int M, K, N;
  float threshold;       // already clamped to >= 0
  const int8_t* Wq;
  const float* w_scale;
  const __half* W16;     // nullable: the layer's fp16 weights [N, K] for the outlier term
  const __half* bias;
  __half* Y;
  int32_t* acc;          // nullable: also write the int32 accumulators
  int splits;            // CTAs per cluster, each owning a K-slice
  int stages;            // depth of the Wq ring
  int per_tensor;        // one activation scale for all rows (the largest row absmax)
  TraceSink trace;       // diagnostic outputs (int8_linear_forward_trace)
  int32_t* status;
};
struct SmallPlan {
  int tiles, splits, kb_per_split, stages;
};
SmallPlan plan_small(int M, int N, int K);
bool small_path_fits(int M, int K);
cudaError_t launch_small(const CUtensorMap& map_wq, const SmallArgs& a, const SmallPlan& p,
                         cudaStream_t stream, bool pdl);

struct GemvArgs {
  const __half* X;
  int M, K, N;
  float threshold;       // already clamped to >= 0
  const int8_t* Wq;
  const float* w_scale;
  const __half* W16;     // nullable: the layer's fp16 weights [N, K] for the outlier term
  const __half* bias;
  __half* Y;
  int32_t* acc;          // nullable: also write the int32 accumulators
  int channels;          // output channels per CTA
  int stages;            // depth of the Wq ring (256-byte slabs of K)
  int kpad;              // K rounded up to 256
  int quant_ctas;        // CTAs (one cluster) of the activation-quantization kernel
  int8_t* xq;            // [16][kpad] int8 activations (written by the quantization kernel)
  __half* xo;            // [n_out][16] fp16 activations of the outlier columns
  float* sx;             // [16] row scales
  int32_t* cols;         // [K] outlier columns, ascending
  int32_t* n_out;        // outlier count
  int per_tensor;        // one activation scale for all rows (the largest row absmax)
  TraceSink trace;       // diagnostic outputs (int8_linear_forward_trace)
  int32_t* status;
};
struct GemvPlan {
  int mt, channels, ctas, kpad, stages, quant_ctas;
  bool fits;
};
GemvPlan plan_gemv(int M, int N, int K, int num_sms);
cudaError_t launch_few_quant(const GemvArgs& a, const GemvPlan& p, cudaStream_t stream, bool pdl);
cudaError_t launch_gemv(const CUtensorMap& map_wq, const GemvArgs& a, const GemvPlan& p,
                        cudaStream_t stream, bool pdl);
int device_sm_count();

// Statistics of |X| (stats.cu): column absmax (nullable), and out[3] = {max, q99, ratio}
// (device doubles); workspace of stats_workspace_bytes() (the |x| histogram).
size_t stats_workspace_bytes();
// row[j] = fp16(col_absmax[j]) where it exceeds the threshold (already clamped to >= 0), else 0
cudaError_t launch_outlier_row(const float* col_absmax, int K, float threshold, __half* row,
                               cudaStream_t stream);
cudaError_t launch_activation_stats(const __half* X, int M, int K, float* col_absmax,
                                    double* out, void* workspace, int num_sms,
                                    cudaStream_t stream);

// One-launch layer for M <= 8 tokens (decode.cu): no workspace.
struct DecodeArgs {
  const __half* X;
  int M, K, N;
  float threshold;       // already clamped to >= 0
  const int8_t* Wq;
  const float* w_scale;
  const __half* W16;     // nullable: the layer's fp16 weights [N, K] for the outlier term
  const __half* bias;
  __half* Y;
  int32_t* acc;          // nullable: also write the int32 accumulators
  int per_tensor;        // one activation scale for all rows (the largest row absmax)
  TraceSink trace;       // diagnostic outputs (int8_linear_forward_trace)
  int32_t* status;
};
struct DecodePlan {
  int tiles;             // 16-channel tiles per CTA (the kernel's T)
  int ctas;
  size_t smem;
  bool fits;
};
DecodePlan plan_decode(int M, int N, int K);
cudaError_t launch_decode(const CUtensorMap& map_wq, const DecodeArgs& a, const DecodePlan& p,
                          cudaStream_t stream, bool pdl);

struct GemmArgs {
  int M, N, K;
  const float* xscale;   // [M]
  const float* w_scale;  // [N]
  const __half* bias;    // [N] or null
  __half* Y;             // fused epilogue output [M,N], or null
  int32_t* C;            // raw int32 accumulators [M,N], or null (at least one of Y, C)
  const int32_t* n_out;  // device outlier count, or null for none
  int group_m;           // row tiles per group of the tile order (set by launch_gemm)
  int bn;                // output channels per tile of the single-CTA product (multiple of 16,
                         // 128..kBN; 0 means kBN), chosen by gemm_tile_width
  int32_t* status;
};
struct GemmMaps {
  CUtensorMap xq, wq, xo, wo;
};
// Host-side tensor-map encoding (driver entry point fetched through the runtime).
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                    uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                    uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);
// 3-D map: dims[0] innermost; strides_bytes[i] is the byte stride of dims[i + 1].
bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                    const uint64_t (&dims)[3], const uint64_t (&strides_bytes)[2],
                    const uint32_t (&box)[3], CUtensorMapSwizzle swizzle);
cudaError_t launch_gemm(const GemmMaps& maps, const GemmArgs& a, cudaStream_t stream, bool pdl);
// Output channels per tile of the single-CTA product for an M x N output: the width (a multiple
// of 16 from 128 to kBN) that minimises (waves of tiles over the persistent CTAs) x (width + a
// fixed per-tile cost), preferring the widest on ties.  The weight maps take boxes of this
// many rows.
int gemm_tile_width(int M, int N);
// The same product with one 256 x 256 tile per CTA pair (gemm2.cu), for M > kPairMinRows; its
// weight maps (wq, wo) take boxes of 128 rows, half of kBN.
cudaError_t launch_gemm_pair(const GemmMaps& maps, const GemmArgs& a, cudaStream_t stream,
                             bool pdl);
constexpr int kPairMinRows = 128;
constexpr int kPairHalfRows = 128;

// GEMM tile shape (shared with the host for map boxes)
constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBKBytes = 128;  // one 128-byte swizzle row: 128 int8 or 64 fp16 per stage

}  // namespace i8mm
