// trace.cu -- the outputs of the diagnostic int8_linear_forward_trace that are gathered after
// the forward's own kernels ran: the ascending outlier-column list built from the outlier bits
// a kernel left behind, and the fp16 outlier weights of the tiled path scattered from their
// compacted operand back to their columns.  Off the hot path.
#include "kernels.cuh"

namespace i8mm {

namespace {

constexpr int kListThreads = 1024;
constexpr int kListWords = INT8MM_MAX_K / 32 / kListThreads;  // mask words per thread

// One block: outlier bits (one per column, little-endian 32-bit words) -> the columns in
// ascending order and their count.  Bits of columns >= K are ignored.
__global__ void __launch_bounds__(kListThreads)
    trace_cols_kernel(const uint32_t* __restrict__ mask, int K, int32_t* __restrict__ cols,
                      int32_t* __restrict__ n_out) {
  __shared__ int warp_sum[kListThreads / 32];
  const int words = (K + 31) / 32;
  const int w0 = threadIdx.x * kListWords;
  uint32_t m[kListWords];
  int local = 0;
#pragma unroll
  for (int u = 0; u < kListWords; ++u) {
    const int w = w0 + u;
    m[u] = 0u;
    if (w < words) {
      m[u] = mask[w];
      if (w == words - 1 && (K & 31)) m[u] &= (1u << (K & 31)) - 1u;
    }
    local += __popc(m[u]);
  }
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int base = 0, total = 0;
  for (int w = 0; w < kListThreads / 32; ++w) {
    base += w < warp ? warp_sum[w] : 0;
    total += warp_sum[w];
  }
  int r = base + incl - local;
  if (cols) {
#pragma unroll
    for (int u = 0; u < kListWords; ++u)
      for (uint32_t b = m[u]; b; b &= b - 1u) cols[r++] = (w0 + u) * 32 + __ffs(b) - 1;
  }
  if (threadIdx.x == 0 && n_out) *n_out = total;
}

// W_hat[n, cols[r]] = wo[n, r] for r < *n_out (the compacted outlier weights of the tiled path).
__global__ void trace_what_kernel(const __half* __restrict__ wo, int ldo,
                                  const int32_t* __restrict__ cols,
                                  const int32_t* __restrict__ n_out_ptr, int N, int K,
                                  __half* __restrict__ W_hat) {
  const int n_out = *n_out_ptr;
  if (n_out <= 0 || n_out > K) return;
  const long long total = static_cast<long long>(N) * n_out;
  for (long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(u / n_out), r = static_cast<int>(u % n_out);
    W_hat[static_cast<size_t>(n) * K + cols[r]] = wo[static_cast<size_t>(n) * ldo + r];
  }
}

}  // namespace

cudaError_t launch_trace_cols(const uint32_t* mask, int K, int32_t* cols, int32_t* n_out,
                              cudaStream_t stream) {
  trace_cols_kernel<<<1, kListThreads, 0, stream>>>(mask, K, cols, n_out);
  return cudaGetLastError();
}

cudaError_t launch_trace_what(const __half* wo, int ldo, const int32_t* cols,
                              const int32_t* n_out, int N, int K, __half* W_hat,
                              cudaStream_t stream) {
  trace_what_kernel<<<2 * device_sm_count(), 256, 0, stream>>>(wo, ldo, cols, n_out, N, K, W_hat);
  return cudaGetLastError();
}

}  // namespace i8mm
