// api.cu -- the extern "C" entry points of libint8mm.so (declared in include/int8mm.h):
// argument checks, workspace carving, tensor-map encoding and kernel launches.  No entry
// point allocates memory or synchronizes, except int8_read_device_status (documented).
#include <cmath>
#include <cstdint>
#include <mutex>

#include "kernels.cuh"

using namespace i8mm;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

int check_shape(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0 || K > INT8MM_MAX_K) return INT8MM_ERR_SHAPE;
  if (K % 16 != 0) return INT8MM_ERR_ALIGN;
  return INT8MM_OK;
}

// The kernels are built for sm_100a only.
int check_device() {
  static int checked_device = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return INT8MM_ERR_CUDA;
  if (dev == checked_device) return INT8MM_OK;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return INT8MM_ERR_CUDA;
  if (major != 10 || minor != 0) return INT8MM_ERR_DEVICE;
  checked_device = dev;
  return INT8MM_OK;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? INT8MM_OK : INT8MM_ERR_CUDA; }

}  // namespace

int i8mm::device_sm_count() {
  static int cached_device = -1, cached_sms = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev != cached_device) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
      sms = 148;
    cached_sms = sms;
    cached_device = dev;
  }
  return cached_sms;
}

namespace {

float effective_threshold(float t) { return t < 0.0f ? 0.0f : t; }

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

}  // namespace

extern "C" {

const char* int8_status_string(int status) {
  switch (status) {
    case INT8MM_OK: return "ok";
    case INT8MM_ERR_NULL: return "a required pointer is NULL";
    case INT8MM_ERR_SHAPE: return "M, N or K out of range";
    case INT8MM_ERR_ALIGN: return "K is not a multiple of 16 or a pointer is not 16-byte aligned";
    case INT8MM_ERR_THRESHOLD: return "threshold is NaN";
    case INT8MM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case INT8MM_ERR_CUDA: return "CUDA runtime or launch error";
    case INT8MM_ERR_DEVICE: return "the current device is not sm_100";
    case INT8MM_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case INT8MM_ERR_OVERFLOW: return "outlier count out of range";
    case INT8MM_ERR_SCRATCH:
      return "the shape needs more scratch than the library's static buffer holds";
    case INT8MM_ERR_FLAGS: return "unknown flag bits";
    default: return "unknown status";
  }
}

int int8_quant_weight(const void* W, int N, int K, int8_t* Wq, float* w_scale,
                      int8mm_stream_t stream) {
  if (!W || !Wq || !w_scale) return INT8MM_ERR_NULL;
  int rc = check_shape(1, N, K);
  if (rc) return rc;
  if (!aligned16(W) || !aligned16(Wq) || !aligned16(w_scale)) return INT8MM_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_status(launch_quant_weight(static_cast<const __half*>(W), N, K, Wq, w_scale,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

size_t int8_linear_workspace_size(int M, int N, int K) {
  if (check_shape(M, N, K) != INT8MM_OK) return 0;
  return workspace_layout(M, N, K).total;
}

}  // extern "C"

namespace {

// Options of the layer beyond its operands: the kept fp16 weights (nullable) and one
// activation scale for the whole of X instead of one per row.
struct LayerOpts {
  const void* W16 = nullptr;
  int per_tensor = 0;
  bool pair_tiles = false;  // M > 128: the products on CTA pairs (gemm2.cu)
  TraceSink trace;  // diagnostic outputs written by the kernels themselves (all null normally)
};

// Which kernels a forward of this shape runs (the dispatch of run_quantize / run_matmul).
enum class Route { kDecode, kGemv, kSmall, kTiled };
Route route_of(int M, int N, int K) {
  if (M <= kSmallMP) {
    if (plan_decode(M, N, K).fits) return Route::kDecode;
    if (plan_gemv(M, N, K, device_sm_count()).fits) return Route::kGemv;
    if (small_path_fits(M, K)) return Route::kSmall;
  }
  return Route::kTiled;
}

struct ForwardPlan {
  WorkspaceLayout L;
  int32_t* header;
  uint32_t* mask;
  int8_t* xq;
  float* xscale;
  __half* xo;
  __half* wo;
};

int plan_forward(int M, int N, int K, const int8_t* Wq, const float* w_scale, void* workspace,
                 size_t ws_bytes, ForwardPlan& p) {
  if (!Wq || !w_scale) return INT8MM_ERR_NULL;
  int rc = check_shape(M, N, K);
  if (rc) return rc;
  if (!aligned16(Wq) || !aligned16(w_scale)) return INT8MM_ERR_ALIGN;
  p.L = workspace_layout(M, N, K);
  if (!workspace || !aligned256(workspace) || ws_bytes < p.L.total) return INT8MM_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  p.header = at<int32_t>(workspace, p.L.header);
  p.mask = at<uint32_t>(workspace, p.L.mask);
  p.xq = at<int8_t>(workspace, p.L.xq);
  p.xscale = at<float>(workspace, p.L.xscale);
  p.xo = at<__half>(workspace, p.L.xo);
  p.wo = at<__half>(workspace, p.L.wo);
  return INT8MM_OK;
}

GemvArgs gemv_args(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
                   const void* bias, int N, float threshold, void* Y, int32_t* acc,
                   void* workspace, const ForwardPlan& p, const GemvPlan& gp,
                   const LayerOpts& o = LayerOpts()) {
  GemvArgs g;
  g.W16 = static_cast<const __half*>(o.W16);
  g.per_tensor = o.per_tensor;
  g.X = static_cast<const __half*>(X);
  g.M = M;
  g.K = K;
  g.N = N;
  g.threshold = effective_threshold(threshold);
  g.Wq = Wq;
  g.w_scale = w_scale;
  g.bias = static_cast<const __half*>(bias);
  g.Y = static_cast<__half*>(Y);
  g.acc = acc;
  g.channels = gp.channels;
  g.stages = gp.stages;
  g.kpad = gp.kpad;
  g.quant_ctas = gp.quant_ctas;
  g.xq = at<int8_t>(workspace, p.L.few_xq);
  g.xo = at<__half>(workspace, p.L.few_xo);
  g.sx = at<float>(workspace, p.L.few_sx);
  g.cols = at<int32_t>(workspace, p.L.cols);
  g.n_out = p.header + 1;
  g.trace = o.trace;
  g.status = p.header;
  return g;
}

SmallArgs small_args(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
                     const void* bias, int N, float threshold, void* Y, int32_t* acc,
                     const ForwardPlan& p, const SmallPlan& sp,
                     const LayerOpts& o = LayerOpts()) {
  SmallArgs a;
  a.W16 = static_cast<const __half*>(o.W16);
  a.per_tensor = o.per_tensor;
  a.X = static_cast<const __half*>(X);
  a.M = M;
  a.K = K;
  a.N = N;
  a.threshold = effective_threshold(threshold);
  a.Wq = Wq;
  a.w_scale = w_scale;
  a.bias = static_cast<const __half*>(bias);
  a.Y = static_cast<__half*>(Y);
  a.acc = acc;
  a.splits = sp.splits;
  a.stages = sp.stages;
  a.trace = o.trace;
  a.status = p.header;
  return a;
}

// The one-launch few-token layer: Wq viewed as [K/128 k-blocks][N rows][128 bytes], one box
// is 16 rows x every k-block, each k-block landing as a 128-byte-swizzled 16 x 128 tile.
int run_decode(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
               const void* bias, int N, float threshold, void* Y, int32_t* acc, int32_t* status,
               const DecodePlan& dp, cudaStream_t stream, bool pdl,
               const LayerOpts& o = LayerOpts()) {
  CUtensorMap map;
  const uint64_t dims[3] = {128, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 128)};
  const uint64_t strides[2] = {static_cast<uint64_t>(K), 128};
  const uint32_t box[3] = {128, 16, static_cast<uint32_t>(K / 128)};
  if (!encode_tmap_3d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return INT8MM_ERR_CUDA;
  DecodeArgs a;
  a.X = static_cast<const __half*>(X);
  a.M = M;
  a.K = K;
  a.N = N;
  a.threshold = effective_threshold(threshold);
  a.Wq = Wq;
  a.w_scale = w_scale;
  a.W16 = static_cast<const __half*>(o.W16);
  a.bias = static_cast<const __half*>(bias);
  a.Y = static_cast<__half*>(Y);
  a.acc = acc;
  a.per_tensor = o.per_tensor;
  a.trace = o.trace;
  a.status = status;
  return launch_status(launch_decode(map, a, dp, stream, pdl));
}

int run_quantize(const void* X, int M, int K, const int8_t* Wq, const float* w_scale, int N,
                 float threshold, void* workspace, const ForwardPlan& p, cudaStream_t stream,
                 bool pdl_first, const LayerOpts& o = LayerOpts()) {
  if (M <= kSmallMP) {
    if (plan_decode(M, N, K).fits) return INT8MM_OK;  // one kernel does everything
    const GemvPlan gp = plan_gemv(M, N, K, device_sm_count());
    if (gp.fits) {
      const GemvArgs g = gemv_args(X, M, K, Wq, w_scale, nullptr, N, threshold, nullptr, nullptr,
                                   workspace, p, gp, o);
      return launch_status(launch_few_quant(g, gp, stream, pdl_first));
    }
    if (small_path_fits(M, K)) return INT8MM_OK;  // one kernel does everything: see run_matmul
  }
  float* word_max = o.per_tensor ? at<float>(workspace, p.L.wmax) : nullptr;
  int rc = launch_status(launch_colmask(static_cast<const __half*>(X), M, K,
                                        effective_threshold(threshold), p.mask, word_max, stream,
                                        pdl_first));
  if (rc) return rc;
  RowQuantArgs rq;
  rq.X = static_cast<const __half*>(X);
  rq.M = M;
  rq.K = K;
  rq.mask = p.mask;
  rq.xq = p.xq;
  rq.xscale = p.xscale;
  rq.xo = p.xo;
  rq.ldo = p.L.ldo;
  rq.cols = at<int32_t>(workspace, p.L.cols);
  rq.n_out = p.header + 1;
  rq.Wq = Wq;
  rq.w_scale = w_scale;
  rq.W16 = static_cast<const __half*>(o.W16);
  rq.wo = p.wo;
  rq.N = N;
  rq.word_max = word_max;
  rq.status = p.header;
  return launch_status(launch_rowquant(rq, stream, true));
}

int run_matmul(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
               const void* bias, int N, float threshold, void* Y, int32_t* acc,
               void* workspace, const ForwardPlan& p, cudaStream_t stream, bool pdl,
               const LayerOpts& o = LayerOpts()) {
  if (M <= kSmallMP) {
    const DecodePlan dp = plan_decode(M, N, K);
    if (dp.fits)
      return run_decode(X, M, K, Wq, w_scale, bias, N, threshold, Y, acc, p.header, dp, stream,
                        pdl, o);
    const GemvPlan gp = plan_gemv(M, N, K, device_sm_count());
    if (gp.fits) {
      const GemvArgs g = gemv_args(X, M, K, Wq, w_scale, bias, N, threshold, Y, acc, workspace,
                                   p, gp, o);
      // Wq viewed as [K/128 k-blocks][N rows][128 bytes]: one box is 32 rows x 8 k-blocks,
      // each k-block landing as a 128-byte-swizzled 32 x 128 tile
      CUtensorMap map;
      const uint64_t dims[3] = {128, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 128)};
      const uint64_t strides[2] = {static_cast<uint64_t>(K), 128};
      const uint32_t box[3] = {128, static_cast<uint32_t>(gp.channels), 8};
      if (!encode_tmap_3d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_128B))
        return INT8MM_ERR_CUDA;
      return launch_status(launch_gemv(map, g, gp, stream, pdl));
    }
  }
  if (small_path_fits(M, K)) {
    const SmallPlan sp = plan_small(M, N, K);
    const SmallArgs a = small_args(X, M, K, Wq, w_scale, bias, N, threshold, Y, acc, p, sp, o);
    CUtensorMap map;
    if (!encode_tmap_2d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, K, N, K, kBKBytes, kSmallBN))
      return INT8MM_ERR_CUDA;
    return launch_status(launch_small(map, a, sp, stream, pdl));
  }
  // on request, many rows: one 256 x 256 tile per CTA pair, each CTA loading 128 weight rows
  const bool pair = o.pair_tiles && M > kPairMinRows;
  const int bn = pair ? kBN : gemm_tile_width(M, N);  // channels per product tile
  const uint32_t wrows = pair ? kPairHalfRows : static_cast<uint32_t>(bn);
  GemmMaps maps;
  if (!encode_tmap_2d(&maps.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.xq, K, M, K, kBKBytes, kBM) ||
      !encode_tmap_2d(&maps.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, K, N, K, kBKBytes, wrows) ||
      !encode_tmap_2d(&maps.xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.xo, p.L.ldo, M,
                      p.L.ldo * 2ull, kBKBytes / 2, kBM) ||
      !encode_tmap_2d(&maps.wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.wo, p.L.ldo, N,
                      p.L.ldo * 2ull, kBKBytes / 2, wrows))
    return INT8MM_ERR_CUDA;
  GemmArgs g;
  g.M = M;
  g.N = N;
  g.K = K;
  g.xscale = p.xscale;
  g.w_scale = w_scale;
  g.bias = static_cast<const __half*>(bias);
  g.Y = static_cast<__half*>(Y);
  g.C = acc;
  g.n_out = p.header + 1;
  g.group_m = 0;
  g.bn = bn;
  g.status = p.header;
  return launch_status(pair ? launch_gemm_pair(maps, g, stream, pdl)
                            : launch_gemm(maps, g, stream, pdl));
}

int forward_impl(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
                 const void* bias, int N, float threshold, void* Y, int32_t* acc,
                 void* workspace, size_t ws_bytes, cudaStream_t stream,
                 const LayerOpts& o = LayerOpts()) {
  if (!X || !Y) return INT8MM_ERR_NULL;
  if (!aligned16(X) || !aligned16(Y) || (bias && !aligned16(bias)) || (acc && !aligned16(acc)) ||
      (o.W16 && !aligned16(o.W16)))
    return INT8MM_ERR_ALIGN;
  if (std::isnan(threshold)) return INT8MM_ERR_THRESHOLD;
  ForwardPlan p;
  int rc = plan_forward(M, N, K, Wq, w_scale, workspace, ws_bytes, p);
  if (rc) return rc;
  if ((rc = run_quantize(X, M, K, Wq, w_scale, N, threshold, workspace, p, stream, true, o)))
    return rc;
  return run_matmul(X, M, K, Wq, w_scale, bias, N, threshold, Y, acc, workspace, p, stream, true,
                    o);
}

}  // namespace

extern "C" {

int int8_linear_forward(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
                        const void* bias, int N, float threshold, void* Y, void* workspace,
                        size_t ws_bytes, int8mm_stream_t stream) {
  return forward_impl(X, M, K, Wq, w_scale, bias, N, threshold, Y, nullptr, workspace, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

int int8_linear_forward_fp16w(const void* X, int M, int K, const int8_t* Wq,
                              const float* w_scale, const void* W16, const void* bias, int N,
                              float threshold, void* Y, void* workspace, size_t ws_bytes,
                              int8mm_stream_t stream) {
  if (!W16) return INT8MM_ERR_NULL;
  LayerOpts o;
  o.W16 = W16;
  return forward_impl(X, M, K, Wq, w_scale, bias, N, threshold, Y, nullptr, workspace, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), o);
}

size_t int8_activation_stats_workspace_size(void) { return stats_workspace_bytes(); }

int int8_activation_stats(const void* X, int M, int K, float* col_absmax, double* out,
                          void* workspace, size_t ws_bytes, int8mm_stream_t stream) {
  if (!X || !out) return INT8MM_ERR_NULL;
  int rc = check_shape(M, 1, K);
  if (rc) return rc;
  if (static_cast<long long>(M) * K >= (1ll << 32)) return INT8MM_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(out) || (col_absmax && !aligned16(col_absmax)))
    return INT8MM_ERR_ALIGN;
  if (!workspace || !aligned256(workspace) || ws_bytes < stats_workspace_bytes())
    return INT8MM_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  return launch_status(launch_activation_stats(static_cast<const __half*>(X), M, K, col_absmax,
                                               out, workspace, device_sm_count(),
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int int8_outlier_row(const float* col_absmax, int K, float threshold, void* row,
                     int8mm_stream_t stream) {
  if (!col_absmax || !row) return INT8MM_ERR_NULL;
  int rc = check_shape(1, 1, K);
  if (rc) return rc;
  if (!aligned16(col_absmax) || !aligned16(row)) return INT8MM_ERR_ALIGN;
  if (std::isnan(threshold)) return INT8MM_ERR_THRESHOLD;
  if ((rc = check_device())) return rc;
  return launch_status(launch_outlier_row(col_absmax, K, effective_threshold(threshold),
                                          static_cast<__half*>(row),
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int int8_linear_forward_ex(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
                           const void* W16, const void* bias, int N, float threshold,
                           unsigned flags, void* Y, int32_t* acc, void* workspace,
                           size_t ws_bytes, int8mm_stream_t stream) {
  if (flags & ~static_cast<unsigned>(INT8MM_PER_TENSOR_SCALE | INT8MM_PAIR_TILES))
    return INT8MM_ERR_FLAGS;
  LayerOpts o;
  o.W16 = W16;
  o.per_tensor = (flags & INT8MM_PER_TENSOR_SCALE) ? 1 : 0;
  o.pair_tiles = (flags & INT8MM_PAIR_TILES) != 0;
  return forward_impl(X, M, K, Wq, w_scale, bias, N, threshold, Y, acc, workspace, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), o);
}

int int8_linear_forward_acc(const void* X, int M, int K, const int8_t* Wq,
                            const float* w_scale, const void* bias, int N, float threshold,
                            void* Y, int32_t* acc, void* workspace, size_t ws_bytes,
                            int8mm_stream_t stream) {
  if (!acc) return INT8MM_ERR_NULL;
  return forward_impl(X, M, K, Wq, w_scale, bias, N, threshold, Y, acc, workspace, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

int int8_linear_quantize(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
                         int N, float threshold, void* workspace, size_t ws_bytes,
                         int8mm_stream_t stream) {
  if (!X) return INT8MM_ERR_NULL;
  if (!aligned16(X)) return INT8MM_ERR_ALIGN;
  if (std::isnan(threshold)) return INT8MM_ERR_THRESHOLD;
  ForwardPlan p;
  int rc = plan_forward(M, N, K, Wq, w_scale, workspace, ws_bytes, p);
  if (rc) return rc;
  return run_quantize(X, M, K, Wq, w_scale, N, threshold, workspace, p,
                      reinterpret_cast<cudaStream_t>(stream), true);
}

int int8_linear_matmul(const void* X, int M, int K, const int8_t* Wq, const float* w_scale,
                       const void* bias, int N, float threshold, void* Y, void* workspace,
                       size_t ws_bytes, int8mm_stream_t stream) {
  if (!X || !Y) return INT8MM_ERR_NULL;
  if (!aligned16(X) || !aligned16(Y) || (bias && !aligned16(bias))) return INT8MM_ERR_ALIGN;
  if (std::isnan(threshold)) return INT8MM_ERR_THRESHOLD;
  ForwardPlan p;
  int rc = plan_forward(M, N, K, Wq, w_scale, workspace, ws_bytes, p);
  if (rc) return rc;
  return run_matmul(X, M, K, Wq, w_scale, bias, N, threshold, Y, nullptr, workspace, p,
                    reinterpret_cast<cudaStream_t>(stream), true);
}

int int8_quantize_rows(const void* X, int M, int K, float threshold, int8_t* Xq,
                       float* row_scale, int32_t* outlier_cols, int32_t* n_outliers,
                       void* workspace, size_t ws_bytes, int8mm_stream_t stream_) {
  if (!X || !Xq || !row_scale || !outlier_cols || !n_outliers) return INT8MM_ERR_NULL;
  int rc = check_shape(M, 1, K);
  if (rc) return rc;
  if (!aligned16(X) || !aligned16(Xq)) return INT8MM_ERR_ALIGN;
  if (std::isnan(threshold)) return INT8MM_ERR_THRESHOLD;
  const WorkspaceLayout L = workspace_layout(M, 1, K);
  if (!workspace || !aligned256(workspace) || ws_bytes < L.total) return INT8MM_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  uint32_t* mask = at<uint32_t>(workspace, L.mask);
  if ((rc = launch_status(launch_colmask(static_cast<const __half*>(X), M, K,
                                         effective_threshold(threshold), mask, nullptr, stream,
                                         false))))
    return rc;
  RowQuantArgs rq = {};
  rq.X = static_cast<const __half*>(X);
  rq.M = M;
  rq.K = K;
  rq.mask = mask;
  rq.xq = Xq;
  rq.xscale = row_scale;
  rq.xo = nullptr;
  rq.ldo = L.ldo;
  rq.cols = outlier_cols;
  rq.n_out = n_outliers;
  rq.wo = nullptr;
  rq.status = at<int32_t>(workspace, L.header);
  return launch_status(launch_rowquant(rq, stream, true));
}

int int8_gemm_i32(const int8_t* Xq, const int8_t* Wq, int M, int N, int K, int32_t* C,
                  int32_t* dev_status, int8mm_stream_t stream_) {
  if (!Xq || !Wq || !C || !dev_status) return INT8MM_ERR_NULL;
  int rc = check_shape(M, N, K);
  if (rc) return rc;
  if (!aligned16(Xq) || !aligned16(Wq) || !aligned16(C)) return INT8MM_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  const bool pair = false;  // the raw product runs on single-CTA tiles
  const int bn = gemm_tile_width(M, N);
  GemmMaps maps;
  if (!encode_tmap_2d(&maps.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, K, M, K, kBKBytes, kBM) ||
      !encode_tmap_2d(&maps.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, K, N, K, kBKBytes,
                      static_cast<uint32_t>(bn)))
    return INT8MM_ERR_CUDA;
  maps.xo = maps.xq;  // unused: no outlier columns
  maps.wo = maps.wq;
  GemmArgs g = {};
  g.M = M;
  g.N = N;
  g.K = K;
  g.C = C;
  g.n_out = nullptr;
  g.bn = bn;
  g.status = dev_status;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  return launch_status(pair ? launch_gemm_pair(maps, g, stream, false)
                            : launch_gemm(maps, g, stream, false));
}

int int8_outlier_weights(const int8_t* Wq, const float* w_scale, int N, int K,
                         const int32_t* outlier_cols, const int32_t* n_outliers, void* W_hat,
                         int8mm_stream_t stream) {
  if (!Wq || !w_scale || !outlier_cols || !n_outliers || !W_hat) return INT8MM_ERR_NULL;
  int rc = check_shape(1, N, K);
  if (rc) return rc;
  if (!aligned16(Wq) || !aligned16(W_hat)) return INT8MM_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_status(launch_outlier_weights(Wq, w_scale, N, K, outlier_cols, n_outliers,
                                              static_cast<__half*>(W_hat),
                                              reinterpret_cast<cudaStream_t>(stream)));
}

int int8_linear_forward_trace(const void* X, int M, int K, const int8_t* Wq,
                              const float* w_scale, const void* W16, const void* bias, int N,
                              float threshold, unsigned flags, void* Y, int32_t* acc, int8_t* Xq,
                              float* row_scale, int32_t* outlier_cols, int32_t* n_outliers,
                              void* W_hat, void* workspace, size_t ws_bytes,
                              int8mm_stream_t stream_) {
  if (flags & ~static_cast<unsigned>(INT8MM_PER_TENSOR_SCALE | INT8MM_PAIR_TILES))
    return INT8MM_ERR_FLAGS;
  if ((Xq && !aligned16(Xq)) || (row_scale && !aligned16(row_scale)) ||
      (outlier_cols && !aligned16(outlier_cols)) || (n_outliers && !aligned16(n_outliers)) ||
      (W_hat && !aligned16(W_hat)))
    return INT8MM_ERR_ALIGN;
  int rc = check_shape(M, N, K);
  if (rc) return rc;
  if (!workspace || !aligned256(workspace) || ws_bytes < workspace_layout(M, N, K).total)
    return INT8MM_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const WorkspaceLayout L = workspace_layout(M, N, K);
  uint32_t* mask = at<uint32_t>(workspace, L.mask);
  const Route route = route_of(M, N, K);
  LayerOpts o;
  o.W16 = W16;
  o.per_tensor = (flags & INT8MM_PER_TENSOR_SCALE) ? 1 : 0;
  o.pair_tiles = (flags & INT8MM_PAIR_TILES) != 0;
  if (route == Route::kDecode || route == Route::kSmall) {
    // these kernels keep codes, scales and outlier bits on chip: they write them out here
    o.trace.xq = Xq;
    o.trace.sx = row_scale;
    o.trace.flags = reinterpret_cast<uint8_t*>(mask);
  }
  if (route != Route::kTiled) o.trace.what = static_cast<__half*>(W_hat);
  if ((rc = forward_impl(X, M, K, Wq, w_scale, bias, N, threshold, Y, acc, workspace, ws_bytes,
                         stream, o)))
    return rc;
  int32_t* header = at<int32_t>(workspace, L.header);
  if (route == Route::kDecode || route == Route::kSmall) {
    if (outlier_cols || n_outliers)
      return launch_status(launch_trace_cols(mask, K, outlier_cols, n_outliers, stream));
    return INT8MM_OK;
  }
  // the other kernels left codes, scales and the outlier list in the workspace
  const bool few = route == Route::kGemv;
  const int8_t* src_xq = at<int8_t>(workspace, few ? L.few_xq : L.xq);
  const size_t src_ld = few ? static_cast<size_t>((K + 255) / 256) * 256 : static_cast<size_t>(K);
  cudaError_t e = cudaSuccess;
  if (Xq)
    e = cudaMemcpy2DAsync(Xq, K, src_xq, src_ld, K, M, cudaMemcpyDeviceToDevice, stream);
  if (e == cudaSuccess && row_scale)
    e = cudaMemcpyAsync(row_scale, at<float>(workspace, few ? L.few_sx : L.xscale),
                        static_cast<size_t>(M) * sizeof(float), cudaMemcpyDeviceToDevice, stream);
  if (e == cudaSuccess && outlier_cols)
    e = cudaMemcpyAsync(outlier_cols, at<int32_t>(workspace, L.cols),
                        static_cast<size_t>(K) * sizeof(int32_t), cudaMemcpyDeviceToDevice, stream);
  if (e == cudaSuccess && n_outliers)
    e = cudaMemcpyAsync(n_outliers, header + 1, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                        stream);
  if (e == cudaSuccess && W_hat && !few)
    e = launch_trace_what(at<__half>(workspace, L.wo), L.ldo, at<int32_t>(workspace, L.cols),
                          header + 1, N, K, static_cast<__half*>(W_hat), stream);
  return launch_status(e);
}

int int8_read_device_status(const int32_t* dev_status, int8mm_stream_t stream) {
  if (!dev_status) return INT8MM_ERR_NULL;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return INT8MM_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, dev_status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
    return INT8MM_ERR_CUDA;
  return v;
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc forward
//
// int8_linear_forward_noalloc serves callers that cannot allocate device memory at the
// point of the call -- code running while a stream is being captured, under an allocator
// that must not grow, or behind a C interface with no workspace argument.  Its scratch (the
// few-token kernels' outlier list, int8 activations, outlier activations and row scales)
// lives in one file-scope device array that every GPU loading the library holds until exit.
// Every call on a device shares it and it keeps the last call's contents.

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[INT8MM_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kNoallocMaxDevices];

// Device address of this device's copy of g_noalloc_scratch, looked up once per device with
// that device current (the host-side name is only a handle for the runtime).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return INT8MM_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return INT8MM_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return INT8MM_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return INT8MM_OK;
}

// The few-token kernels' regions, carved from the scratch: status header, outlier list,
// 16-row int8 activations, outlier activations, row scales (the same regions and sizes as
// the few-token part of workspace_layout; the other regions are not used on this path).
WorkspaceLayout noalloc_layout(int K) {
  WorkspaceLayout L = {};
  L.ldo = (K + 63) / 64 * 64;
  const size_t kpad = static_cast<size_t>((K + 255) / 256) * 256;
  size_t off = 0;
  L.header = off;  off = align256(off + 64 * sizeof(int32_t));
  L.cols = off;    off = align256(off + static_cast<size_t>(K) * sizeof(int32_t));
  L.few_xq = off;  off = align256(off + kSmallMP * kpad);
  L.few_xo = off;  off = align256(off + static_cast<size_t>(K) * kSmallMP * sizeof(__half));
  L.few_sx = off;  off = align256(off + kSmallMP * sizeof(float));
  L.mask = L.xscale = L.xq = L.xo = L.wo = L.header;
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

int int8_linear_forward_noalloc(const void* X, int M, int K, const int8_t* Wq,
                                const float* w_scale, const void* bias, int N, float threshold,
                                void* Y, int32_t* dev_status, int8mm_stream_t stream_) {
  if (!X || !Y || !Wq || !w_scale) return INT8MM_ERR_NULL;
  int rc = check_shape(M, N, K);
  if (rc) return rc;
  if (!aligned16(X) || !aligned16(Y) || !aligned16(Wq) || !aligned16(w_scale) ||
      (bias && !aligned16(bias)) || (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)))
    return INT8MM_ERR_ALIGN;
  if (std::isnan(threshold)) return INT8MM_ERR_THRESHOLD;
  if (M > kSmallMP) return INT8MM_ERR_SCRATCH;
  if ((rc = check_device())) return rc;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const DecodePlan dp = plan_decode(M, N, K);
  if (dp.fits)  // the one-launch kernel needs no scratch
    return run_decode(X, M, K, Wq, w_scale, bias, N, threshold, Y, nullptr, dev_status, dp,
                      stream, true);
  const GemvPlan gp = plan_gemv(M, N, K, device_sm_count());
  const bool small = !gp.fits && small_path_fits(M, K);
  if (!gp.fits && !small) return INT8MM_ERR_SCRATCH;
  const WorkspaceLayout L = noalloc_layout(K);
  ForwardPlan p = {};
  p.L = L;
  p.header = at<int32_t>(scratch, L.header);
  // Nothing in the scratch has to start at zero: the quantization kernel writes the outlier
  // count, list and activations before the product kernel reads them, and the status goes to
  // the caller's word (or nowhere).
  if (small) {  // the cluster kernel keeps everything on chip: no scratch, no size limit
    const SmallPlan sp = plan_small(M, N, K);
    SmallArgs a = small_args(X, M, K, Wq, w_scale, bias, N, threshold, Y, nullptr, p, sp);
    a.status = dev_status;
    CUtensorMap map;
    if (!encode_tmap_2d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, K, N, K, kBKBytes, kSmallBN))
      return INT8MM_ERR_CUDA;
    return launch_status(launch_small(map, a, sp, stream, true));
  }
  if (L.total > INT8MM_NOALLOC_SCRATCH_BYTES) return INT8MM_ERR_SCRATCH;
  GemvArgs g = gemv_args(X, M, K, Wq, w_scale, bias, N, threshold, Y, nullptr, scratch, p, gp);
  g.status = dev_status;
  CUtensorMap map;
  const uint64_t dims[3] = {128, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 128)};
  const uint64_t strides[2] = {static_cast<uint64_t>(K), 128};
  const uint32_t box[3] = {128, static_cast<uint32_t>(gp.channels), 8};
  if (!encode_tmap_3d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return INT8MM_ERR_CUDA;
  if ((rc = launch_status(launch_few_quant(g, gp, stream, true)))) return rc;
  return launch_status(launch_gemv(map, g, gp, stream, true));
}

}  // extern "C"
