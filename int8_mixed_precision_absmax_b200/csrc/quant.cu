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
// Quantization arithmetic: scale = absmax / 127 and q = x / scale are IEEE float32 quotients
// (__fdiv_rn; in the row pass the quotient comes from one correction of x * RN(1/scale), equal
// to it), q is rounded to nearest with ties to even and lies in [-127, 127].  Absolute maxima
// are taken on the binary16 values (exact).
#include "codes.cuh"
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
// A cluster of 8 CTAs owns a strip of 64 columns; CTA r of the cluster takes rows
// r, r + 8, ...: thread (l, c) = (tid / 8, tid % 8) reads the 16-byte chunk c of the strip in
// 8 of those rows at a time (all 8 loads in flight; one batch covers M <= 2048).  Each CTA reduces its column maxima
// (fp16, exact) into its shared memory; after one cluster barrier CTA 0 takes the maximum over
// the 8 CTAs through distributed shared memory and writes the strip's two mask words.  No two
// clusters write the same word, so the mask needs no clearing.

constexpr int kCMThreads = 256;
constexpr int kCMCluster = 8;
constexpr int kCMStrip = 64;                       // columns per cluster
constexpr int kCMRowLanes = kCMThreads / 8;        // 32 row lanes x 8 chunks of 8 columns
constexpr int kCMUnroll = 8;                       // loads in flight per thread

__device__ __forceinline__ uint32_t cm_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__global__ void __launch_bounds__(kCMThreads) colmask_kernel(const __half* __restrict__ X, int M,
                                                             int K, float threshold,
                                                             uint32_t* __restrict__ mask,
                                                             float* __restrict__ word_max) {
  __shared__ __half2 red[kCMThreads / 32][8][4];
  __shared__ __half cmax_local[kCMStrip];  // this CTA's column maxima (read by CTA 0)
  const int strip = blockIdx.x / kCMCluster;
  const int rank = static_cast<int>(cm_cluster_rank());
  const int c = threadIdx.x & 7, l = threadIdx.x >> 3;
  const int col0 = strip * kCMStrip + c * 8;
  // Ask L2 for this CTA's rows of the strip before waiting for the previous launch.  L2 is
  // where global memory is kept coherent, so this is safe even while that launch may still be
  // writing X: its stores land in the same lines, and X is read only after the wait.
  if (strip * kCMStrip < K) {
    const int seg = min(kCMStrip, K - strip * kCMStrip) * 2;  // bytes of the row segment
    for (int i = rank + kCMCluster * threadIdx.x; i < M; i += kCMCluster * kCMThreads)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                       reinterpret_cast<uint64_t>(X + static_cast<size_t>(i) * K + strip * kCMStrip)),
                   "r"(seg)
                   : "memory");
  }
  grid_dependency_wait();
  __half2 m[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) m[e] = __float2half2_rn(0.0f);
  if (col0 < K) {  // K % 8 == 0: a chunk is entirely inside or outside the matrix
    // rows i = rank + 8 (l + 32 u): consecutive lanes of a warp read neighbouring chunks
    for (int base = rank + kCMCluster * l; base < M; base += kCMCluster * kCMRowLanes * kCMUnroll) {
      uint4 v[kCMUnroll];
#pragma unroll
      for (int u = 0; u < kCMUnroll; ++u) {
        const int i = base + u * kCMCluster * kCMRowLanes;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (i < M) v[u] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(i) * K + col0));
      }
#pragma unroll
      for (int u = 0; u < kCMUnroll; ++u) {
        m[0] = habs2_max(m[0], v[u].x);
        m[1] = habs2_max(m[1], v[u].y);
        m[2] = habs2_max(m[2], v[u].z);
        m[3] = habs2_max(m[3], v[u].w);
      }
    }
  }
  grid_launch_dependents();
  // reduce over the 4 row lanes of the warp (lanes with equal c), then across warps
#pragma unroll
  for (int e = 0; e < 4; ++e) {
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) m[e] = __hmax2(m[e], __shfl_xor_sync(0xffffffffu, m[e], o));
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane < 8) {
#pragma unroll
    for (int e = 0; e < 4; ++e) red[warp][lane][e] = m[e];
  }
  __syncthreads();
  if (threadIdx.x < kCMStrip) {  // thread j: column 64 strip + j
    const int j = threadIdx.x, cg = j / 8, ce = (j % 8) / 2, hi = j % 2;
    __half h = __float2half_rn(0.0f);
#pragma unroll
    for (int w = 0; w < kCMThreads / 32; ++w) {
      const __half2 v = red[w][cg][ce];
      h = __hmax(h, hi ? __high2half(v) : __low2half(v));
    }
    cmax_local[j] = h;
  }
  __syncthreads();
  // warp 0 releases the CTA's shared-memory writes for all threads (cumulative); every warp
  // arrives with one instruction
  if (warp == 0) asm volatile("barrier.cluster.arrive.release;" ::: "memory");
  else asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
  if (rank == 0 && threadIdx.x < kCMStrip) {  // whole warps 0, 1
    const uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(&cmax_local[threadIdx.x]));
    unsigned short hv[kCMCluster];
#pragma unroll
    for (int q = 0; q < kCMCluster; ++q) {
      uint32_t remote;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(q));
      asm volatile("ld.shared::cluster.u16 %0, [%1];" : "=h"(hv[q]) : "r"(remote));
    }
    float cm = 0.0f;
#pragma unroll
    for (int q = 0; q < kCMCluster; ++q) cm = fmaxf(cm, __half2float(__ushort_as_half(hv[q])));
    const uint32_t bits = __ballot_sync(0xffffffffu, cm > threshold);
    const int word = strip * 2 + threadIdx.x / 32;
    if (lane == 0 && word * 32 < K) mask[word] = bits;
    if (word_max) {  // the largest |x| of the word's regular columns (columns past K hold 0)
      float rm = cm > threshold ? 0.0f : cm;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, o));
      if (lane == 0 && word * 32 < K) word_max[word] = rm;
    }
  }
  // no CTA leaves while CTA 0 may still read its shared memory
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

cudaError_t launch_colmask(const __half* X, int M, int K, float threshold, uint32_t* mask,
                           float* word_max, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(((K + kCMStrip - 1) / kCMStrip) * kCMCluster);
  cfg.blockDim = dim3(kCMThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCMCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, colmask_kernel, X, M, K, threshold, mask, word_max);
}

// ------------------------------------------------------------------ rows + outlier operands
//
// The row pass.  A block of 256 threads takes rpb rows at a time (rpb = 1, 2, 4 or 8, so that
// a thread owns about 8 chunks of 8 columns or more) with tpr = 256 / rpb threads per row (a
// template parameter): thread (row t / tpr, lane t % tpr) owns chunks lane + tpr j of its row.
// It stages its own chunks in shared memory with 16-byte asynchronous copies and is their only
// reader, so the staging needs no block barrier and holds no registers; as soon as a chunk is
// quantized its slot is refilled with the same chunk of the block's next row.  Blocks are persistent (up to
// four per SM) and read the outlier mask and its prefix once.  Per row:
//   1. outlier columns: their fp16 values to X_O at their compacted index, then 0 in the stage,
//      so that the absolute maximum below is the regular columns' and their codes come out 0;
//   2. the row's absolute maximum (fp16 maxima of the sign-cleared values, exact): shuffles,
//      then one named barrier across the row's warps;
//   3. codes rne(x / s), the IEEE quotient from packed fp32 FMAs (codes8 in codes.cuh).
// The first row's copies go out before the wait on the column search: X is not written by that
// kernel, and whatever wrote X had completed before the column search let this launch start.
// Before their rows, all blocks write the fp16 outlier weights
// W_hat[n, r] = fp16(Wq[n, col(r)] * w_scale[n]) (or the kept fp16 weight W16[n, col(r)]),
// zero-padded to a multiple of 64, while their first rows land.

constexpr int kRQThreads = 256;
constexpr int kRQWarps = kRQThreads / 32;
constexpr int kRQChunksPerThread = 8;  // rows share a block while a thread keeps this many chunks
constexpr int kRQBlocksPerSM = 4;
constexpr int kGatherCols = 256;       // outlier columns the weight gather lists at a time

struct RowPassSmem {  // byte offsets into the dynamic shared memory
  int words, tpr, rpb, mask, prefix, misc, red, cols, stage, total;
};

__host__ __device__ inline RowPassSmem row_pass_smem(int K) {
  RowPassSmem L;
  L.words = (K + 31) / 32;
  const int chunks = K / 8;
  int rpb = 1;
  while (rpb < 8 && chunks * rpb * 2 <= kRQThreads * kRQChunksPerThread) rpb *= 2;
  L.rpb = rpb;
  L.tpr = kRQThreads / rpb;
  const int wpad = (L.words + 3) / 4 * 4;
  L.mask = 0;
  L.prefix = wpad * 4;
  L.misc = L.prefix + wpad * 4;  // int32 [0] outlier count, [8..15] per-warp sums
  L.red = L.misc + 64;           // float [2][8] per-warp row maxima (two rows in flight)
  L.cols = L.red + 64;           // int32 [kGatherCols]
  L.stage = (L.cols + kGatherCols * 4 + 127) / 128 * 128;
  L.total = L.stage + rpb * K * 2;
  return L;
}

namespace {

// Mask words into shared memory and the exclusive prefix of their popcounts; n_out = total.
__device__ void stage_mask_prefix(const uint32_t* __restrict__ gmask, uint32_t* mask,
                                  int32_t* prefix, int32_t* warp_sum, int32_t* n_out, int words) {
  const int per = (words + kRQThreads - 1) / kRQThreads;
  const int w0 = threadIdx.x * per;
  int local = 0;
  for (int w = w0; w < min(w0 + per, words); ++w) {
    const uint32_t m = gmask[w];
    mask[w] = m;
    local += __popc(m);
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
  int warp_base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kRQWarps; ++w) {
    const int v = warp_sum[w];
    warp_base += (w < warp) ? v : 0;
    total += v;
  }
  int run = warp_base + incl - local;
  for (int w = w0; w < min(w0 + per, words); ++w) {
    prefix[w] = run;
    run += __popc(mask[w]);
  }
  if (threadIdx.x == 0) *n_out = total;
  __syncthreads();
}

// The fp16 values of chunk c's outlier columns (bits), at their places in the compacted row.
__device__ __forceinline__ void emit_outliers(const uint32_t* mask, const int32_t* prefix,
                                              const uint4& x, int c, uint32_t bits, __half* xo) {
  const int word = c >> 2;
  const uint32_t wm = mask[word];
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int e = 0; e < 8; ++e)
    if ((bits >> e) & 1u) {
      const int bit = (c & 3) * 8 + e;
      const int r = prefix[word] + __popc(wm & ((1u << bit) - 1u));
      const uint32_t hb = (w[e / 2] >> (16 * (e & 1))) & 0xFFFFu;
      xo[r] = __ushort_as_half(static_cast<unsigned short>(hb));
    }
}

// Block gb of G: W_hat[n, r] for units (n, group of 8 outliers); the outliers are taken in
// windows of kGatherCols columns listed in shared memory.
__device__ void gather_weights(const RowQuantArgs& a, const uint32_t* mask,
                               const int32_t* prefix, int n_out, int32_t* cols, int words,
                               int gb, int G) {
  const int width = (n_out + 63) / 64 * 64;
  for (int R0 = 0; R0 < width; R0 += kGatherCols) {  // block-uniform
    const int R1 = min(n_out, R0 + kGatherCols);      // outliers of this window
    for (int w = threadIdx.x; w < words; w += kRQThreads) {
      const int p0 = prefix[w];
      uint32_t m = mask[w];
      if (p0 >= R1 || p0 + __popc(m) <= R0) continue;
      for (int r = p0; m; ++r, m &= m - 1)
        if (r >= R0 && r < R1) cols[r - R0] = w * 32 + __ffs(m) - 1;
    }
    __syncthreads();
    const int groups = (min(width, R0 + kGatherCols) - R0) / 8;  // <= 32
    const long long units = static_cast<long long>(a.N) * groups;
    for (long long u = static_cast<long long>(gb) * kRQThreads + threadIdx.x; u < units;
         u += static_cast<long long>(G) * kRQThreads) {
      const int n = static_cast<int>(u / groups);
      const int r0 = R0 + static_cast<int>(u - static_cast<long long>(n) * groups) * 8;
      uint32_t h[4] = {0u, 0u, 0u, 0u};
      // eight outliers in consecutive columns from a multiple of 8 (every column, when the
      // threshold is 0): one vector load of the row instead of eight
      const int c0 = r0 < n_out ? cols[r0 - R0] : 0;
      const bool dense = r0 + 8 <= n_out && (c0 & 7) == 0 && cols[r0 + 7 - R0] == c0 + 7;
      if (dense && a.W16 != nullptr) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.W16 + static_cast<size_t>(n) * a.K + c0));
        h[0] = v.x;
        h[1] = v.y;
        h[2] = v.z;
        h[3] = v.w;
      } else if (dense) {
        const uint2 q = __ldg(reinterpret_cast<const uint2*>(a.Wq + static_cast<size_t>(n) * a.K + c0));
        const float sc = a.w_scale[n];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int8_t code = static_cast<int8_t>(((e < 4 ? q.x : q.y) >> (8 * (e & 3))) & 0xFFu);
          const float w = static_cast<float>(code) * sc;
          h[e / 2] |= static_cast<uint32_t>(__half_as_ushort(__float2half_rn(w))) << (16 * (e & 1));
        }
      } else if (r0 < n_out && a.W16 != nullptr) {  // the layer's own fp16 weights
        const unsigned short* hrow =
            reinterpret_cast<const unsigned short*>(a.W16) + static_cast<size_t>(n) * a.K;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (r0 + e < n_out)
            h[e / 2] |= static_cast<uint32_t>(hrow[cols[r0 + e - R0]]) << (16 * (e & 1));
      } else if (r0 < n_out) {  // rebuilt from the int8 weights
        const float sc = a.w_scale[n];
        const int8_t* wrow = a.Wq + static_cast<size_t>(n) * a.K;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int r = r0 + e;
          if (r < n_out) {
            const float w = static_cast<float>(wrow[cols[r - R0]]) * sc;
            h[e / 2] |= static_cast<uint32_t>(__half_as_ushort(__float2half_rn(w)))
                        << (16 * (e & 1));
          }
        }
      }
      *reinterpret_cast<uint4*>(a.wo + static_cast<size_t>(n) * a.ldo + r0) =
          make_uint4(h[0], h[1], h[2], h[3]);
    }
    __syncthreads();  // the list is rewritten for the next window
  }
}

// Shared memory through 32-bit shared-window addresses.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src))
               : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace

// TPR = threads per row (256, 128, 64 or 32: the block takes 256 / TPR rows at a time).
template <int TPR>
__global__ void __launch_bounds__(kRQThreads, kRQBlocksPerSM) rowquant_kernel(const RowQuantArgs a) {
  constexpr int kRpb = kRQThreads / TPR, kWpr = TPR / 32;  // rows per block, warps per row
  extern __shared__ __align__(128) uint8_t rq_smem[];
  const RowPassSmem L = row_pass_smem(a.K);
  uint32_t* mask = reinterpret_cast<uint32_t*>(rq_smem + L.mask);
  int32_t* prefix = reinterpret_cast<int32_t*>(rq_smem + L.prefix);
  int32_t* misc = reinterpret_cast<int32_t*>(rq_smem + L.misc);
  float* red = reinterpret_cast<float*>(rq_smem + L.red);
  const int K = a.K, M = a.M, chunks = K / 8;
  const int rl = threadIdx.x / TPR, lr = threadIdx.x % TPR;
  // this thread's row stage: chunk c at stage + 16 c (it owns c = lr + TPR j)
  const uint32_t stage = smem_addr(rq_smem + L.stage) + static_cast<uint32_t>(rl * chunks) * 16u;
  const int step = gridDim.x * kRpb;  // rows between a block's consecutive row groups
  int i = blockIdx.x * kRpb + rl;
  if (i < M) {
    const uint4* src = reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * K);
    for (int c = lr; c < chunks; c += TPR) cp_async16(stage + 16u * c, src + c);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  grid_dependency_wait();  // the outlier mask is complete from here on
  stage_mask_prefix(a.mask, mask, prefix, misc + 8, misc, L.words);
  grid_launch_dependents();
  const int n_out = misc[0];
  if (blockIdx.x == 0) {
    for (int w = threadIdx.x; w < L.words; w += kRQThreads) {
      uint32_t m = mask[w];
      int r = prefix[w];
      while (m) {
        a.cols[r++] = w * 32 + __ffs(m) - 1;
        m &= m - 1;
      }
    }
    if (threadIdx.x == 0) *a.n_out = n_out;
  }
  if (a.wo != nullptr)
    gather_weights(a, mask, prefix, n_out, reinterpret_cast<int32_t*>(rq_smem + L.cols), L.words,
                   blockIdx.x, gridDim.x);
  float tensor_max = -1.0f;  // one scale for all rows: the largest regular |x| of the tensor
  if (a.word_max) {
    float g = 0.0f;
    for (int w = threadIdx.x % 32; w < L.words; w += 32) g = fmaxf(g, __ldcg(a.word_max + w));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
    tensor_max = g;
  }
  const uint8_t* bits_of = reinterpret_cast<const uint8_t*>(mask);  // byte c: chunk c's outliers
  // bit j: this thread's chunk lr + TPR j holds an outlier column (at most 32 chunks a thread:
  // K <= 65536 with TPR = 256, and narrower rows have fewer)
  uint32_t ochunks = 0u;
  for (int j = 0, c = lr; c < chunks; ++j, c += TPR)
    if (bits_of[c]) ochunks |= 1u << j;
  const int warp = threadIdx.x / 32;
  // every thread of the block takes the same number of steps (rows past M idle)
  for (int it = 0; blockIdx.x * kRpb + it * step < M; ++it) {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    const bool live = i < M;
    __half* xo = (a.xo && live) ? a.xo + static_cast<size_t>(i) * a.ldo : nullptr;
    __half2 h0 = __float2half2_rn(0.0f), h1 = h0, h2 = h0, h3 = h0;
    if (live) {
      if (ochunks) {  // the outlier columns: to X_O, then 0 in the stage
        for (int j = 0, c = lr; c < chunks; ++j, c += TPR) {
          if (!((ochunks >> j) & 1u)) continue;
          const uint32_t bits = bits_of[c];
          const uint4 x = lds128(stage + 16u * c);
          if (xo) emit_outliers(mask, prefix, x, c, bits, xo);
          uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if ((bits >> e) & 1u) w[e / 2] &= (e & 1) ? 0x0000FFFFu : 0xFFFF0000u;
          sts128(stage + 16u * c, make_uint4(w[0], w[1], w[2], w[3]));
        }
      }
#pragma unroll 4
      for (int c = lr; c < chunks; c += TPR) {
        const uint4 x = lds128(stage + 16u * c);
        uint32_t b0 = x.x & 0x7FFF7FFFu, b1 = x.y & 0x7FFF7FFFu, b2 = x.z & 0x7FFF7FFFu,
                 b3 = x.w & 0x7FFF7FFFu;
        h0 = __hmax2(h0, *reinterpret_cast<const __half2*>(&b0));
        h1 = __hmax2(h1, *reinterpret_cast<const __half2*>(&b1));
        h2 = __hmax2(h2, *reinterpret_cast<const __half2*>(&b2));
        h3 = __hmax2(h3, *reinterpret_cast<const __half2*>(&b3));
      }
      if (xo != nullptr) {
        const int padded = (n_out + 63) / 64 * 64;
        for (int r = n_out + lr; r < padded; r += TPR) xo[r] = __float2half_rn(0.0f);
      }
    }
    float amax = half2_max_f(__hmax2(__hmax2(h0, h1), __hmax2(h2, h3)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if constexpr (kWpr > 1) {  // across the row's warps; two buffers, as a warp may be one row ahead
      float* rd = red + (it & 1) * kRQWarps;
      if ((threadIdx.x & 31) == 0) rd[warp] = amax;
      named_barrier(1 + rl, TPR);
#pragma unroll
      for (int w = 0; w < kWpr; ++w) amax = fmaxf(amax, rd[rl * kWpr + w]);
    }
    if (tensor_max >= 0.0f) amax = tensor_max;
    const int nx = i + step;
    if (live) {
      const float s = __fdiv_rn(amax, 127.0f);
      if (lr == 0) a.xscale[i] = s;
      const float rcp = amax == 0.0f ? 0.0f : __frcp_rn(s);
      uint2* out = reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(i) * K);
      if (nx < M) {  // each slot is refilled with the next row's chunk once its codes are out
        const uint4* next = reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(nx) * K);
#pragma unroll 4
        for (int c = lr; c < chunks; c += TPR) {
          const uint4 x = lds128(stage + 16u * c);
          out[c] = codes8(x, s, rcp);
          cp_async16(stage + 16u * c, next + c);
        }
      } else {
#pragma unroll 4
        for (int c = lr; c < chunks; c += TPR) out[c] = codes8(lds128(stage + 16u * c), s, rcp);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    i = nx;
  }
}

cudaError_t launch_rowquant(const RowQuantArgs& a, cudaStream_t stream, bool pdl) {
  // per device: shared memory of an SM, reserved per block, and the opt-in set on the kernel
  constexpr int kMaxDevices = 64;
  static int smem_per_sm[kMaxDevices] = {}, reserved[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (smem_per_sm[dev] == 0) {
    int optin = 0, res = 0, per_sm_bytes = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&res, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&per_sm_bytes, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    for (const void* k : {reinterpret_cast<const void*>(rowquant_kernel<256>),
                          reinterpret_cast<const void*>(rowquant_kernel<128>),
                          reinterpret_cast<const void*>(rowquant_kernel<64>),
                          reinterpret_cast<const void*>(rowquant_kernel<32>)})
      if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    reserved[dev] = res;
    smem_per_sm[dev] = per_sm_bytes;
  }
  const RowPassSmem L = row_pass_smem(a.K);
  int per_sm = smem_per_sm[dev] / (L.total + reserved[dev]);
  if (per_sm > kRQBlocksPerSM) per_sm = kRQBlocksPerSM;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  long long want = (a.M + L.rpb - 1) / L.rpb;
  if (a.wo != nullptr) {  // enough blocks for the weight gather (worst case: every column)
    const long long units = static_cast<long long>(a.N) * (a.ldo / 8);
    const long long gather = (units + kRQThreads - 1) / kRQThreads;
    const long long cap = 2LL * device_sm_count();
    const long long g = gather < cap ? gather : cap;
    if (g > want) want = g;
  }
  const long long resident = static_cast<long long>(per_sm) * device_sm_count();
  const int blocks = static_cast<int>(want < resident ? want : resident);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kRQThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  switch (L.tpr) {
    case 256: return cudaLaunchKernelEx(&cfg, rowquant_kernel<256>, a);
    case 128: return cudaLaunchKernelEx(&cfg, rowquant_kernel<128>, a);
    case 64: return cudaLaunchKernelEx(&cfg, rowquant_kernel<64>, a);
    default: return cudaLaunchKernelEx(&cfg, rowquant_kernel<32>, a);
  }
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
