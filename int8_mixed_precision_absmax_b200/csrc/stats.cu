// stats.cu -- statistics of |X| for choosing the outlier threshold ([P2] "8位量化实战：离群值
// 处理与显存优化避坑指南" section 5.1: the largest |x|, its 0.99 quantile and their ratio; and
// the absmax of every column, which is what the threshold is compared against).
//
// |x| of a binary16 value is its bit pattern without the sign, and those 32768 patterns order
// as the values do, so a histogram with one bin per pattern holds the exact order statistics:
// the quantile needs no sort.  Two launches:
//   * stats_hist_kernel: CTA (chunk group, row group) reads 32 chunks of 8 columns over its
//     rows; each thread keeps the column maxima of its chunk and counts its values into a
//     shared-memory histogram, which is added into the global one (non-empty bins only); the
//     column maxima meet in shared memory and go to the global column absmax with atomicMax
//     (non-negative floats order as their bit patterns do).
//   * stats_finish_kernel (one CTA): prefix sums over the bins find the values of rank lo and
//     lo + 1, lo = floor(0.99 (n - 1)), and q99 = v_lo + (0.99 (n - 1) - lo) (v_hi - v_lo) in
//     double; max is the highest non-empty bin; ratio = max / (q99 + 1e-6).
#include "kernels.cuh"

namespace i8mm {

namespace {

constexpr int kStBins = 32768;
constexpr int kStThreads = 512;
constexpr int kStChunks = 32;                       // 8-column chunks per CTA
constexpr int kStRowLanes = kStThreads / kStChunks;  // 16 threads per chunk walk the rows
constexpr int kFinThreads = 1024;
constexpr int kFinBinsPerThread = kStBins / kFinThreads;  // 32

__global__ void __launch_bounds__(kStThreads, 1)
    stats_hist_kernel(const __half* __restrict__ X, int M, int K, int rows_per_cta,
                      uint32_t* __restrict__ hist, float* __restrict__ col_absmax) {
  extern __shared__ uint32_t st_hist[];                    // kStBins counters
  __shared__ uint32_t colmax[kStRowLanes][kStChunks * 8];  // |x| bits, per row lane
  for (int b = threadIdx.x; b < kStBins; b += kStThreads) st_hist[b] = 0u;
  __syncthreads();
  const int chunk = blockIdx.x * kStChunks + threadIdx.x % kStChunks;
  const int lane_row = threadIdx.x / kStChunks;
  const int r0 = blockIdx.y * rows_per_cta;
  const int r1 = min(M, r0 + rows_per_cta);
  uint32_t cm[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  if (chunk * 8 < K) {
    for (int i = r0 + lane_row; i < r1; i += kStRowLanes) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(i) * K) + chunk);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t a = (w[e / 2] >> (16 * (e & 1))) & 0x7FFFu;
        atomicAdd(&st_hist[a], 1u);
        cm[e] = max(cm[e], a);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) colmax[lane_row][(threadIdx.x % kStChunks) * 8 + e] = cm[e];
  __syncthreads();
  if (col_absmax && threadIdx.x < kStChunks * 8) {  // column 8 chunk + e of the CTA
    const int j = blockIdx.x * kStChunks * 8 + threadIdx.x;
    uint32_t m = 0u;
#pragma unroll
    for (int l = 0; l < kStRowLanes; ++l) m = max(m, colmax[l][threadIdx.x]);
    if (j < K) {
      const float f = __half2float(__ushort_as_half(static_cast<unsigned short>(m)));
      atomicMax(reinterpret_cast<unsigned int*>(col_absmax + j), __float_as_uint(f));
    }
  }
  for (int b = threadIdx.x; b < kStBins; b += kStThreads) {
    const uint32_t c = st_hist[b];
    if (c) atomicAdd(hist + b, c);
  }
}

__device__ __forceinline__ double bin_value(int b) {
  return static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(b))));
}

__global__ void __launch_bounds__(kFinThreads, 1)
    stats_finish_kernel(const uint32_t* __restrict__ hist, long long n, double* __restrict__ out) {
  __shared__ unsigned long long part[kFinThreads];
  __shared__ int found[2];
  __shared__ int top;
  const int t = threadIdx.x;
  if (t == 0) {
    found[0] = found[1] = 0;
    top = 0;
  }
  unsigned long long mine = 0ull;
  int hi_bin = -1;
  for (int u = 0; u < kFinBinsPerThread; ++u) {
    const uint32_t c = hist[t * kFinBinsPerThread + u];
    mine += c;
    if (c) hi_bin = t * kFinBinsPerThread + u;
  }
  part[t] = mine;
  __syncthreads();
  if (hi_bin >= 0) atomicMax(&top, hi_bin);
  // inclusive scan of the per-thread sums (Hillis-Steele over 1024 entries)
  for (int o = 1; o < kFinThreads; o <<= 1) {
    const unsigned long long add = t >= o ? part[t - o] : 0ull;
    __syncthreads();
    part[t] += add;
    __syncthreads();
  }
  const double pos = 0.99 * static_cast<double>(n - 1);
  const long long lo = static_cast<long long>(floor(pos));
  const long long want[2] = {lo, lo + 1 < n ? lo + 1 : lo};
  unsigned long long before = t ? part[t - 1] : 0ull;  // values in bins below this thread's
  for (int u = 0; u < kFinBinsPerThread; ++u) {
    const int b = t * kFinBinsPerThread + u;
    const unsigned long long c = hist[b];
#pragma unroll
    for (int q = 0; q < 2; ++q)
      if (c && static_cast<unsigned long long>(want[q]) >= before &&
          static_cast<unsigned long long>(want[q]) < before + c)
        found[q] = b;
    before += c;
  }
  __syncthreads();
  if (t == 0) {
    const double a = bin_value(found[0]), b = bin_value(found[1]);
    const double q99 = a + (pos - static_cast<double>(lo)) * (b - a);
    const double mx = bin_value(top);
    out[0] = mx;
    out[1] = q99;
    out[2] = mx / (q99 + 1e-6);
  }
}

}  // namespace

size_t stats_workspace_bytes() { return static_cast<size_t>(kStBins) * sizeof(uint32_t); }

cudaError_t launch_activation_stats(const __half* X, int M, int K, float* col_absmax,
                                    double* out, void* workspace, int num_sms,
                                    cudaStream_t stream) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int smem = kStBins * static_cast<int>(sizeof(uint32_t));
  if (dev != configured_device) {
    e = cudaFuncSetAttribute(stats_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  uint32_t* hist = static_cast<uint32_t*>(workspace);
  if ((e = cudaMemsetAsync(hist, 0, stats_workspace_bytes(), stream)) != cudaSuccess) return e;
  if (col_absmax &&
      (e = cudaMemsetAsync(col_absmax, 0, static_cast<size_t>(K) * sizeof(float), stream)) !=
          cudaSuccess)
    return e;
  const int groups = (K / 8 + kStChunks - 1) / kStChunks;
  int row_groups = (2 * num_sms + groups - 1) / groups;
  row_groups = max(1, min(row_groups, M));
  const int rows_per_cta = (M + row_groups - 1) / row_groups;
  row_groups = (M + rows_per_cta - 1) / rows_per_cta;
  stats_hist_kernel<<<dim3(groups, row_groups), kStThreads, smem, stream>>>(X, M, K, rows_per_cta,
                                                                             hist, col_absmax);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  stats_finish_kernel<<<1, kFinThreads, 0, stream>>>(hist, static_cast<long long>(M) * K, out);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ the token split's row

// row[j] = binary16(col_absmax[j]) where col_absmax[j] > threshold, else 0: one row that
// exceeds the threshold in exactly the columns whose maximum over all rows does (the outlier
// test of [P2] section 2.3, in float32 as in every kernel of the layer).
__global__ void outlier_row_kernel(const float* __restrict__ col_absmax, int K, float threshold,
                                   __half* __restrict__ row) {
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < K; j += gridDim.x * blockDim.x) {
    const float c = col_absmax[j];
    row[j] = c > threshold ? __float2half_rn(c) : __float2half_rn(0.0f);
  }
}

cudaError_t launch_outlier_row(const float* col_absmax, int K, float threshold, __half* row,
                               cudaStream_t stream) {
  const int blocks = (K + 255) / 256;
  outlier_row_kernel<<<blocks, 256, 0, stream>>>(col_absmax, K, threshold, row);
  return cudaGetLastError();
}

}  // namespace i8mm
