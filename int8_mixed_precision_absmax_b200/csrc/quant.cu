// quant.cu -- the HBM-bound quantization passes of the LLM.int8() layer.
//
//   quant_weight_kernel  per-output-channel weight quantization (once, at load time)
//                        [P5] "PyTorch 2.9 支持 LLM.int8()" section "LLM.int8() 是怎么做到
//                        几乎无损的", item 1
//   colmask_kernel       outlier feature columns: max_i |X[i,j]| > threshold
//                        [P2] "8位量化实战：离群值处理与显存优化避坑指南" section 2.3
//   rowquant_kernel      per-row absmax over the regular columns, scale, int8 codes, and
//                        the compacted fp16 operands of the outlier term (activations by
//                        row blocks, fp16(Wq*w_scale) weights by extra blocks)
//                        [P5] item 2 and item 3; [P2] section 2.3
//
// Quantization arithmetic: scale = absmax / 127 and q = x / scale are IEEE float32
// divisions (__fdiv_rn), q is rounded to nearest with ties to even (__float2int_rn) and
// clamped to [-127, 127].  Absolute maxima are taken on the binary16 values (exact).
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

__device__ __forceinline__ int quantize_value(float x, float s) {
  const int q = __float2int_rn(__fdiv_rn(x, s));
  return max(-127, min(127, q));
}

__device__ __forceinline__ __half2 habs2_max(__half2 m, uint32_t bits) {
  __half2 v = *reinterpret_cast<__half2*>(&bits);
  return __hmax2(m, __habs2(v));
}

__device__ __forceinline__ float half2_max_f(__half2 m) {
  return fmaxf(__low2float(m), __high2float(m));
}

template <int NT>
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();  // red may still be in use by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = (lane < NT / 32) ? red[lane] : 0.0f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 8 halves (one 16-byte chunk) -> 8 int8 codes packed little-endian into 8 bytes.
__device__ __forceinline__ uint2 quantize_chunk(uint4 v, float s, bool zero_all,
                                                uint32_t outlier_bits) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t hb = (w[e / 2] >> (16 * (e & 1))) & 0xFFFFu;
    const float x = __half2float(__ushort_as_half(static_cast<unsigned short>(hb)));
    int q = 0;
    if (!zero_all && !((outlier_bits >> e) & 1u)) q = quantize_value(x, s);
    packed[e / 4] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (e & 3));
  }
  return make_uint2(packed[0], packed[1]);
}

}  // namespace

// ------------------------------------------------------------------ weights (once)

constexpr int kQWThreads = 256;

__global__ void __launch_bounds__(kQWThreads) quant_weight_kernel(const __half* __restrict__ W,
                                                                  int K,
                                                                  int8_t* __restrict__ Wq,
                                                                  float* __restrict__ w_scale) {
  __shared__ float red[kQWThreads / 32];
  const int n = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(W + static_cast<size_t>(n) * K);
  const int chunks = K / 8;
  __half2 m2 = __float2half2_rn(0.0f);
  for (int c = threadIdx.x; c < chunks; c += kQWThreads) {
    const uint4 v = __ldg(row + c);
    m2 = habs2_max(m2, v.x);
    m2 = habs2_max(m2, v.y);
    m2 = habs2_max(m2, v.z);
    m2 = habs2_max(m2, v.w);
  }
  const float a = block_max<kQWThreads>(half2_max_f(m2), red);
  const float s = __fdiv_rn(a, 127.0f);
  if (threadIdx.x == 0) w_scale[n] = s;
  uint2* out = reinterpret_cast<uint2*>(Wq + static_cast<size_t>(n) * K);
  for (int c = threadIdx.x; c < chunks; c += kQWThreads)
    out[c] = quantize_chunk(__ldg(row + c), s, a == 0.0f, 0u);
}

cudaError_t launch_quant_weight(const __half* W, int N, int K, int8_t* Wq, float* w_scale,
                                cudaStream_t stream) {
  quant_weight_kernel<<<N, kQWThreads, 0, stream>>>(W, K, Wq, w_scale);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ outlier columns
//
// One block owns 32 consecutive columns (one mask word) for all M rows, so no two blocks
// write the same word and the mask needs no atomics and no prior clearing.  Thread
// (r, g) = (tid / 4, tid % 4) reads the 16-byte chunk of columns [32b + 8g, +8) of rows
// r, r + 64, ...; the per-column maxima are then reduced across the 64 row lanes.

constexpr int kCMThreads = 256;
constexpr int kCMRowLanes = kCMThreads / 4;
constexpr int kCMUnroll = 8;

__global__ void __launch_bounds__(kCMThreads) colmask_kernel(const __half* __restrict__ X, int M,
                                                             int K, float threshold,
                                                             uint32_t* __restrict__ mask) {
  __shared__ __half2 red[kCMThreads / 32][4][4];
  grid_dependency_wait();
  const int g = threadIdx.x & 3, r = threadIdx.x >> 2;
  const int col0 = blockIdx.x * 32 + g * 8;
  __half2 m[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) m[e] = __float2half2_rn(0.0f);
  if (col0 < K) {  // K % 8 == 0: a chunk is entirely inside or outside the matrix
    const __half* base = X + col0;
    int i = r;
    for (; i + (kCMUnroll - 1) * kCMRowLanes < M; i += kCMUnroll * kCMRowLanes) {
      uint4 v[kCMUnroll];
#pragma unroll
      for (int u = 0; u < kCMUnroll; ++u)
        v[u] = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(i + u * kCMRowLanes) * K));
#pragma unroll
      for (int u = 0; u < kCMUnroll; ++u) {
        m[0] = habs2_max(m[0], v[u].x);
        m[1] = habs2_max(m[1], v[u].y);
        m[2] = habs2_max(m[2], v[u].z);
        m[3] = habs2_max(m[3], v[u].w);
      }
    }
    for (; i < M; i += kCMRowLanes) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(i) * K));
      m[0] = habs2_max(m[0], v.x);
      m[1] = habs2_max(m[1], v.y);
      m[2] = habs2_max(m[2], v.z);
      m[3] = habs2_max(m[3], v.w);
    }
  }
  grid_launch_dependents();
  // reduce over the 8 row lanes inside the warp (lanes with equal g), then across warps
#pragma unroll
  for (int e = 0; e < 4; ++e) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      const __half2 other = __shfl_xor_sync(0xffffffffu, m[e], o);
      m[e] = __hmax2(m[e], other);
    }
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane < 4) {
#pragma unroll
    for (int e = 0; e < 4; ++e) red[warp][lane][e] = m[e];
  }
  __syncthreads();
  if (warp == 0) {
    // lane c owns column 32b + c: chunk g = c / 8, half2 e = (c % 8) / 2, half (c % 2)
    const int cg = lane / 8, ce = (lane % 8) / 2, hi = lane % 2;
    float cmax = 0.0f;
#pragma unroll
    for (int w = 0; w < kCMThreads / 32; ++w) {
      const __half2 v = red[w][cg][ce];
      cmax = fmaxf(cmax, hi ? __high2float(v) : __low2float(v));
    }
    const uint32_t bits = __ballot_sync(0xffffffffu, cmax > threshold);
    if (lane == 0) mask[blockIdx.x] = bits;
  }
}

cudaError_t launch_colmask(const __half* X, int M, int K, float threshold, uint32_t* mask,
                           cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((K + 31) / 32);
  cfg.blockDim = dim3(kCMThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, colmask_kernel, X, M, K, threshold, mask);
}

// ------------------------------------------------------------------ rows + outlier operands

constexpr int kRQThreads = 256;
constexpr int kRQRegChunks = 8;                         // chunks of 8 halves kept per thread
constexpr int kRQRegK = kRQThreads * 8 * kRQRegChunks;  // rows up to this length stay in registers
constexpr int kRQMaxWords = INT8MM_MAX_K / 32;

struct RowQuantShared {
  uint32_t mask[kRQMaxWords];
  int32_t prefix[kRQMaxWords];  // outliers in the words before this one
  int32_t warp_sum[kRQThreads / 32];
  float red[kRQThreads / 32];
  int32_t n_out;
};

// Load the mask into shared memory and build the exclusive prefix of its popcounts.
__device__ void load_mask_prefix(RowQuantShared& S, const uint32_t* __restrict__ mask, int words) {
  const int per = (words + kRQThreads - 1) / kRQThreads;
  const int w0 = threadIdx.x * per;
  int local = 0;
  for (int w = w0; w < min(w0 + per, words); ++w) {
    const uint32_t m = mask[w];
    S.mask[w] = m;
    local += __popc(m);
  }
  // exclusive scan of `local` over the block
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) S.warp_sum[warp] = incl;
  __syncthreads();
  int warp_base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kRQThreads / 32; ++w) {
    const int v = S.warp_sum[w];
    warp_base += (w < warp) ? v : 0;
    total += v;
  }
  int run = warp_base + incl - local;
  for (int w = w0; w < min(w0 + per, words); ++w) {
    S.prefix[w] = run;
    run += __popc(S.mask[w]);
  }
  if (threadIdx.x == 0) S.n_out = total;
  __syncthreads();
}

// Column of the r-th outlier (0-based, r < n_out): binary search over the prefix table.
__device__ __forceinline__ int outlier_column(const RowQuantShared& S, int words, int r) {
  int lo = 0, hi = words - 1;  // find the last word with prefix <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (S.prefix[mid] <= r) lo = mid; else hi = mid - 1;
  }
  uint32_t m = S.mask[lo];
  for (int k = r - S.prefix[lo]; k > 0; --k) m &= m - 1u;  // drop the lower outliers
  return lo * 32 + __ffs(m) - 1;
}

// Block for one row: absmax over the regular columns, scale, codes, outlier activations.
__device__ void quantize_row(const RowQuantArgs& a, RowQuantShared& S, int i) {
  const int K = a.K;
  const int chunks = K / 8;
  const uint4* row = reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * K);
  const bool in_regs = K <= kRQRegK;
  uint4 v[kRQRegChunks];
  __half2 m2 = __float2half2_rn(0.0f);
  float mf = 0.0f;
  // pass 1: absmax over regular columns
  auto absmax_chunk = [&](const uint4& x, int c) {
    const uint32_t bits = (S.mask[c >> 2] >> ((c & 3) * 8)) & 0xFFu;
    if (bits == 0) {
      m2 = habs2_max(m2, x.x);
      m2 = habs2_max(m2, x.y);
      m2 = habs2_max(m2, x.z);
      m2 = habs2_max(m2, x.w);
    } else {
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (!((bits >> e) & 1u)) {
          const uint32_t hb = (w[e / 2] >> (16 * (e & 1))) & 0xFFFFu;
          mf = fmaxf(mf, fabsf(__half2float(__ushort_as_half(static_cast<unsigned short>(hb)))));
        }
    }
  };
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kRQRegChunks; ++u) {
      const int c = threadIdx.x + u * kRQThreads;
      if (c < chunks) v[u] = __ldg(row + c);
    }
#pragma unroll
    for (int u = 0; u < kRQRegChunks; ++u) {
      const int c = threadIdx.x + u * kRQThreads;
      if (c < chunks) absmax_chunk(v[u], c);
    }
  } else {
    for (int c = threadIdx.x; c < chunks; c += kRQThreads) absmax_chunk(__ldg(row + c), c);
  }
  const float amax = block_max<kRQThreads>(fmaxf(mf, half2_max_f(m2)), S.red);
  const float s = __fdiv_rn(amax, 127.0f);
  if (threadIdx.x == 0) a.xscale[i] = s;
  const bool zero_row = amax == 0.0f;

  // pass 2: codes and the outlier activations
  uint2* out = reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(i) * K);
  __half* xo = a.xo ? a.xo + static_cast<size_t>(i) * a.ldo : nullptr;
  auto emit_chunk = [&](const uint4& x, int c) {
    const uint32_t bits = (S.mask[c >> 2] >> ((c & 3) * 8)) & 0xFFu;
    out[c] = quantize_chunk(x, s, zero_row, bits);
    if (bits != 0 && xo != nullptr) {
      const int word = c >> 2;
      const uint32_t wm = S.mask[word];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if ((bits >> e) & 1u) {
          const int bit = (c & 3) * 8 + e;
          const int r = S.prefix[word] + __popc(wm & ((1u << bit) - 1u));
          const uint32_t hb = (w[e / 2] >> (16 * (e & 1))) & 0xFFFFu;
          xo[r] = __ushort_as_half(static_cast<unsigned short>(hb));
        }
    }
  };
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kRQRegChunks; ++u) {
      const int c = threadIdx.x + u * kRQThreads;
      if (c < chunks) emit_chunk(v[u], c);
    }
  } else {
    for (int c = threadIdx.x; c < chunks; c += kRQThreads) emit_chunk(__ldg(row + c), c);
  }
  if (xo != nullptr) {
    const int n_out = S.n_out;
    const int padded = (n_out + 63) / 64 * 64;
    for (int r = n_out + threadIdx.x; r < padded; r += kRQThreads) xo[r] = __float2half_rn(0.0f);
  }
}

// Extra blocks: W_hat[n, r] = fp16(float(Wq[n, col(r)]) * w_scale[n]), zero-padded to 64.
__device__ void gather_weights(const RowQuantArgs& a, RowQuantShared& S, int words, int gb,
                               int G) {
  const int n_out = S.n_out;
  const int width = (n_out + 63) / 64 * 64;
  const int groups = width / 8;  // 8 consecutive outliers per thread step (one 16-byte store)
  const long long units = static_cast<long long>(a.N) * groups;
  for (long long u = static_cast<long long>(gb) * kRQThreads + threadIdx.x; u < units;
       u += static_cast<long long>(G) * kRQThreads) {
    const int n = static_cast<int>(u / groups);
    const int r0 = static_cast<int>(u % groups) * 8;
    const float sc = a.w_scale[n];
    const int8_t* wrow = a.Wq + static_cast<size_t>(n) * a.K;
    uint32_t h[4] = {0u, 0u, 0u, 0u};
    if (r0 < n_out) {
      int col = outlier_column(S, words, r0);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int r = r0 + e;
        if (r < n_out) {
          if (e > 0) {  // next set bit after col
            int w = (col + 1) >> 5;
            uint32_t rest = ((col + 1) & 31) ? (S.mask[w] & (~0u << ((col + 1) & 31))) : S.mask[w];
            while (rest == 0) rest = S.mask[++w];
            col = w * 32 + __ffs(rest) - 1;
          }
          const __half hv = __float2half_rn(static_cast<float>(wrow[col]) * sc);
          h[e / 2] |= static_cast<uint32_t>(__half_as_ushort(hv)) << (16 * (e & 1));
        }
      }
    }
    *reinterpret_cast<uint4*>(a.wo + static_cast<size_t>(n) * a.ldo + r0) =
        make_uint4(h[0], h[1], h[2], h[3]);
  }
}

__global__ void __launch_bounds__(kRQThreads) rowquant_kernel(const RowQuantArgs a) {
  extern __shared__ __align__(16) uint8_t rq_smem[];
  RowQuantShared& S = *reinterpret_cast<RowQuantShared*>(rq_smem);
  grid_dependency_wait();
  const int words = (a.K + 31) / 32;
  load_mask_prefix(S, a.mask, words);
  grid_launch_dependents();
  if (blockIdx.x == 0) {
    for (int w = threadIdx.x; w < words; w += kRQThreads) {
      uint32_t m = S.mask[w];
      int r = S.prefix[w];
      while (m) {
        const int b = __ffs(m) - 1;
        a.cols[r++] = w * 32 + b;
        m &= m - 1;
      }
    }
    if (threadIdx.x == 0) *a.n_out = S.n_out;
  }
  if (static_cast<int>(blockIdx.x) < a.M) {
    quantize_row(a, S, blockIdx.x);
  } else if (a.wo != nullptr) {
    gather_weights(a, S, words, blockIdx.x - a.M, gridDim.x - a.M);
  }
}

cudaError_t launch_rowquant(const RowQuantArgs& a, cudaStream_t stream, bool pdl) {
  static bool configured = false;
  const int smem = static_cast<int>(sizeof(RowQuantShared));
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(rowquant_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int gather_blocks = 0;
  if (a.wo != nullptr) {
    const long long worst_units = static_cast<long long>(a.N) * (a.ldo / 8);
    const long long want = (worst_units + kRQThreads - 1) / kRQThreads;
    gather_blocks = static_cast<int>(want < 1184 ? want : 1184);
    if (gather_blocks < 1) gather_blocks = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.M + gather_blocks);
  cfg.blockDim = dim3(kRQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, rowquant_kernel, a);
}

// ------------------------------------------------------------------ diagnostic: W_hat alone

__global__ void outlier_weights_kernel(const int8_t* __restrict__ Wq,
                                       const float* __restrict__ w_scale, int N, int K,
                                       const int32_t* __restrict__ cols,
                                       const int32_t* __restrict__ n_out_ptr,
                                       __half* __restrict__ W_hat) {
  const int n_out = *n_out_ptr;
  if (n_out <= 0 || n_out > K) return;
  const long long total = static_cast<long long>(N) * n_out;
  for (long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(u / n_out), r = static_cast<int>(u % n_out);
    const float w = static_cast<float>(Wq[static_cast<size_t>(n) * K + cols[r]]) * w_scale[n];
    W_hat[static_cast<size_t>(n) * K + r] = __float2half_rn(w);
  }
}

cudaError_t launch_outlier_weights(const int8_t* Wq, const float* w_scale, int N, int K,
                                   const int32_t* cols, const int32_t* n_out, __half* W_hat,
                                   cudaStream_t stream) {
  outlier_weights_kernel<<<1184, 256, 0, stream>>>(Wq, w_scale, N, K, cols, n_out, W_hat);
  return cudaGetLastError();
}

}  // namespace i8mm
