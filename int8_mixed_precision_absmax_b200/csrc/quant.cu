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

// 8 halves -> 8 int8 codes q = rne(x / s) of a row whose regular columns satisfy
// |x| <= absmax = 127 s, packed little-endian, outlier columns (bits) set to 0.
// With r = 1/s rounded to nearest, the exact x * r is within 2^-17 of x / s (|x / s| <= 128)
// and the rounded quotient within 2^-18, so rne(x * r) = rne(fl(x / s)) unless x * r lies
// within 2^-15 of a half-integer; there the quotient itself (__fdiv_rn) is rounded.
// tb = fl(x * r + 1.5 * 2^23) = 1.5 * 2^23 + rne(x * r) exactly, and as 1.5 * 2^23 has a zero
// low byte, the low byte of tb's bits is the two's-complement code.  d = x * r - rne(x * r)
// (one more FMA, rounding error <= 2^-25) has |d| <= 1/2, so "near a half-integer" is
// |d| > 1/2 - 2^-15.  |x / s| <= 127 (1 + 2^-22) on regular columns: no clamp is needed.
__device__ __forceinline__ uint32_t keep_mask(uint32_t bits4) {  // bit e set -> byte e = 0
  return ~(((bits4 * 0x204081u) & 0x01010101u) * 0xFFu);
}
__device__ __forceinline__ uint2 quantize_chunk_fast(const uint4& v, float s, float rcp,
                                                     uint32_t bits) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  constexpr float kNear = 0.5f - 0x1p-15f;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float x[8];
  uint32_t qb[8];
  bool near_tie = false;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e / 2]));
    x[e] = f.x;
    x[e + 1] = f.y;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float tb = __fmaf_rn(x[e], rcp, kRound);
    qb[e] = __float_as_uint(tb);
    const float d = __fmaf_rn(x[e], rcp, -(tb - kRound));
    near_tie |= fabsf(d) > kNear && !((bits >> e) & 1u);
  }
  if (near_tie) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float tb = __fmaf_rn(x[e], rcp, kRound);
      const float d = __fmaf_rn(x[e], rcp, -(tb - kRound));
      if (fabsf(d) > kNear && !((bits >> e) & 1u))
        qb[e] = static_cast<uint32_t>(__float2int_rn(__fdiv_rn(x[e], s)));
    }
  }
  const uint32_t lo = __byte_perm(__byte_perm(qb[0], qb[1], 0x0040), __byte_perm(qb[2], qb[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(qb[4], qb[5], 0x0040), __byte_perm(qb[6], qb[7], 0x0040), 0x5410);
  return make_uint2(lo & keep_mask(bits & 0xFu), hi & keep_mask(bits >> 4));
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
// 16 of those rows at a time (all 16 loads in flight; one batch covers M <= 4096).  Each CTA reduces its column maxima
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

constexpr int kRQThreads = 256;
constexpr int kRQRegChunks = 8;                         // chunks of 8 halves kept per thread
constexpr int kRQRegK = kRQThreads * 8 * kRQRegChunks;  // rows up to this length stay in registers
constexpr int kRQMaxWords = INT8MM_MAX_K / 32;

constexpr int kGatherSmemCols = 2048;  // outlier columns the weight gather lists in smem

struct RowQuantShared {
  uint32_t mask[kRQMaxWords];
  int32_t prefix[kRQMaxWords];  // outliers in the words before this one
  int32_t cols[kGatherSmemCols];  // the outlier columns (weight gather, n_out <= 2048)
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

// The row pass.  A block takes rpb = 256 / tpr rows (tpr = threads per row, 32..256): thread
// (row t / tpr, lane t % tpr) holds chunks lane + u * tpr (u < 8) of its row in registers
// (rows of up to kRQRegK columns), so the block keeps up to 32 KB of X in flight and shares
// one mask prologue.  Longer rows (one per block) are read twice from global memory.

// outlier bits (one per column) of chunk c: byte c % 4 of mask word c / 4
__device__ __forceinline__ uint32_t chunk_bits(const RowQuantShared& S, int c) {
  return (S.mask[c >> 2] >> ((c & 3) * 8)) & 0xFFu;
}

__device__ __forceinline__ void absmax_chunk(const uint4& x, uint32_t bits, __half2& m2, float& mf) {
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
}

// the fp16 values of chunk c's outlier columns, at their places in the compacted row
__device__ __forceinline__ void emit_outliers(const RowQuantShared& S, const uint4& x, int c,
                                              uint32_t bits, __half* xo) {
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

// Row i of the block (tpr threads): absmax over the regular columns, scale, codes, outlier
// activations.  In-register rows arrive in v.
__device__ void quantize_rows_block(const RowQuantArgs& a, RowQuantShared& S, int tpr,
                                    const uint4 (&v)[kRQRegChunks]) {
  const int K = a.K;
  const int chunks = K / 8;
  const int rl = threadIdx.x / tpr, lr = threadIdx.x % tpr;
  const int i = blockIdx.x * (kRQThreads / tpr) + rl;
  const bool live = i < a.M;
  const bool in_regs = K <= kRQRegK;
  const uint4* row = reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(live ? i : 0) * K);
  __half2 m2 = __float2half2_rn(0.0f);
  float mf = 0.0f;
  uint32_t bits_r[kRQRegChunks];
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kRQRegChunks; ++u) {
      const int c = lr + u * tpr;
      bits_r[u] = 0u;
      if (live && c < chunks) {
        bits_r[u] = chunk_bits(S, c);
        absmax_chunk(v[u], bits_r[u], m2, mf);
      }
    }
  } else if (live) {
    for (int c = lr; c < chunks; c += tpr) absmax_chunk(__ldg(row + c), chunk_bits(S, c), m2, mf);
  }
  // maximum over the row's tpr threads: the warp, then the row's warps
  float m = fmaxf(mf, half2_max_f(m2));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int warp = threadIdx.x / 32;
  if ((threadIdx.x & 31) == 0) S.red[warp] = m;
  __syncthreads();
  float amax = 0.0f;
  for (int w = rl * (tpr / 32); w < (rl + 1) * (tpr / 32); ++w) amax = fmaxf(amax, S.red[w]);
  if (a.word_max) {  // one scale for all rows: the largest regular |x| of the whole tensor
    const int lane = threadIdx.x & 31;
    float g = 0.0f;
    for (int w = lane; w < (K + 31) / 32; w += 32) g = fmaxf(g, __ldcg(a.word_max + w));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
    amax = g;
  }
  if (!live) return;
  const float s = __fdiv_rn(amax, 127.0f);
  if (lr == 0) a.xscale[i] = s;
  const bool zero_row = amax == 0.0f;
  const float rcp = zero_row ? 0.0f : __frcp_rn(s);

  uint2* out = reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(i) * K);
  __half* xo = a.xo ? a.xo + static_cast<size_t>(i) * a.ldo : nullptr;
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kRQRegChunks; ++u) {
      const int c = lr + u * tpr;
      if (c < chunks) {
        out[c] = zero_row ? make_uint2(0u, 0u) : quantize_chunk_fast(v[u], s, rcp, bits_r[u]);
        if (bits_r[u] != 0 && xo != nullptr) emit_outliers(S, v[u], c, bits_r[u], xo);
      }
    }
  } else {
    for (int c = lr; c < chunks; c += tpr) {
      const uint4 x = __ldg(row + c);
      const uint32_t bits = chunk_bits(S, c);
      out[c] = zero_row ? make_uint2(0u, 0u) : quantize_chunk_fast(x, s, rcp, bits);
      if (bits != 0 && xo != nullptr) emit_outliers(S, x, c, bits, xo);
    }
  }
  if (xo != nullptr) {
    const int n_out = S.n_out;
    const int padded = (n_out + 63) / 64 * 64;
    for (int r = n_out + lr; r < padded; r += tpr) xo[r] = __float2half_rn(0.0f);
  }
}

// Extra blocks: W_hat[n, r] = fp16(float(Wq[n, col(r)]) * w_scale[n]), zero-padded to 64 (or
// the kept fp16 weight W16[n, col(r)] when the layer has one).
// The outliers are taken in windows of kGatherSmemCols: the block lists the window's columns
// in shared memory, then thread u writes the 8 consecutive entries (one 16-byte store) of
// channel u / groups, group u % groups of the window.
__device__ void gather_weights(const RowQuantArgs& a, RowQuantShared& S, int words, int gb,
                               int G) {
  const int n_out = S.n_out;
  const int width = (n_out + 63) / 64 * 64;
  for (int R0 = 0; R0 < width; R0 += kGatherSmemCols) {  // block-uniform
    const int R1 = min(n_out, R0 + kGatherSmemCols);     // outliers of this window
    for (int w = threadIdx.x; w < words; w += kRQThreads) {
      const int p0 = S.prefix[w];
      uint32_t m = S.mask[w];
      if (p0 >= R1 || p0 + __popc(m) <= R0) continue;
      for (int r = p0; m; ++r, m &= m - 1)
        if (r >= R0 && r < R1) S.cols[r - R0] = w * 32 + __ffs(m) - 1;
    }
    __syncthreads();
    const int groups = (min(width, R0 + kGatherSmemCols) - R0) / 8;
    const long long units = static_cast<long long>(a.N) * groups;
    for (long long u = static_cast<long long>(gb) * kRQThreads + threadIdx.x; u < units;
         u += static_cast<long long>(G) * kRQThreads) {
      const int n = static_cast<int>(u / groups);
      const int r0 = R0 + static_cast<int>(u % groups) * 8;
      uint32_t h[4] = {0u, 0u, 0u, 0u};
      // eight outliers in consecutive columns from a multiple of 8 (every column, when the
      // threshold is 0): one vector load of the row instead of eight
      const int c0 = r0 < n_out ? S.cols[r0 - R0] : 0;
      const bool dense = r0 + 8 <= n_out && (c0 & 7) == 0 && S.cols[r0 + 7 - R0] == c0 + 7;
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
            h[e / 2] |= static_cast<uint32_t>(hrow[S.cols[r0 + e - R0]]) << (16 * (e & 1));
      } else if (r0 < n_out) {  // rebuilt from the int8 weights
        const float sc = a.w_scale[n];
        const int8_t* wrow = a.Wq + static_cast<size_t>(n) * a.K;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int r = r0 + e;
          if (r < n_out) {
            const float w = static_cast<float>(wrow[S.cols[r - R0]]) * sc;
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

// (The row pass is capped at 64 registers, four 256-thread blocks per SM: measured 7% faster on
// prefill up_proj than the 80 the compiler picks alone, equal on the longer rows.)

// threads per row of the row pass: rows of up to 2048 / rpb chunks share a block
__host__ __device__ inline int rowquant_tpr(int K) {
  const int chunks = K / 8;
  int rpb = 1;
  while (rpb < 8 && chunks * rpb * 2 <= kRQThreads * kRQRegChunks) rpb *= 2;
  return kRQThreads / rpb;
}

__global__ void __launch_bounds__(kRQThreads, 4) rowquant_kernel(const RowQuantArgs a, int row_blocks) {
  extern __shared__ __align__(16) uint8_t rq_smem[];
  RowQuantShared& S = *reinterpret_cast<RowQuantShared*>(rq_smem);
  const int words = (a.K + 31) / 32;
  const int tpr = rowquant_tpr(a.K);
  // The rows' loads go out before the wait on the column search: X is not written by that
  // kernel, and whatever wrote X was complete before the column search (which waited for it)
  // let this launch start.
  const bool row_block = static_cast<int>(blockIdx.x) < row_blocks;
  const int chunks = a.K / 8;
  uint4 v[kRQRegChunks];
  if (row_block && a.K <= kRQRegK) {
    const int i = blockIdx.x * (kRQThreads / tpr) + threadIdx.x / tpr, lr = threadIdx.x % tpr;
    const uint4* row = reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * a.K);
#pragma unroll
    for (int u = 0; u < kRQRegChunks; ++u) {
      const int c = lr + u * tpr;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i < a.M && c < chunks) v[u] = __ldg(row + c);
    }
  }
  grid_dependency_wait();  // the outlier mask is complete from here on
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
  if (row_block) {
    quantize_rows_block(a, S, tpr, v);
  } else if (a.wo != nullptr) {
    gather_weights(a, S, words, blockIdx.x - row_blocks, gridDim.x - row_blocks);
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
    const long long cap = 2LL * device_sm_count();
    gather_blocks = static_cast<int>(want < cap ? want : cap);
    if (gather_blocks < 1) gather_blocks = 1;
  }
  const int rpb = kRQThreads / rowquant_tpr(a.K);
  const int row_blocks = (a.M + rpb - 1) / rpb;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(row_blocks + gather_blocks);
  cfg.blockDim = dim3(kRQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, rowquant_kernel, a, row_blocks);
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
