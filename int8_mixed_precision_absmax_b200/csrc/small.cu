// small.cu -- the LLM.int8() layer for a few tokens (M <= 16: the decode regime).
//
// With so few rows the layer is a weight-streaming problem (read Wq once at HBM speed), so
// the 128 x 256 tiles of gemm.cu would leave most SMs idle.  This path uses two kernels:
//
//   small_stats_kernel  one block per 256-column strip of X: the strip's outlier-mask words
//                       ([P2] "8位量化实战：离群值处理与显存优化避坑指南" section 2.3) and, per
//                       row, the maximum |x| over the strip's regular columns (the
//                       vector-wise absmax of [P5] "PyTorch 2.9 支持 LLM.int8()" item 2,
//                       taken over X_R).  All <= 16 rows of a strip live in one block, so
//                       both results are complete per strip: no atomics, no cross-block wait.
//   small_gemm_kernel   swap-AB tensor-core product with split-K.  Each CTA owns 128 output
//                       channels and a slice of K.  Its TMA warp streams the Wq slice before
//                       waiting on the stats kernel (the weights do not depend on it); six
//                       warps meanwhile quantize the CTA's K-slice of X (row scale = max of
//                       the strip maxima / 127, q = rne(x / s), 0 in outlier columns) straight
//                       into the 128-byte-swizzled shared-memory layout of the MMA's B
//                       operand; one thread issues tcgen05.mma kind::i8 (M = 128 channels,
//                       N = 16 tokens, int32 accumulator in TMEM).  The CTA writes its int32
//                       partial sums; the last CTA of a channel tile to finish (an atomic
//                       count it resets itself) adds the partials in split order (exact),
//                       the fp16 outlier term sum_j X[i,j] * fp16(Wq[n,j] * w_scale[n]) and
//                       the bias, and writes Y.  No CTA ever waits for another.
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kThreads = 256;
constexpr int kStripCols = kSmallStrip;
constexpr int kStages = 4;
constexpr int kABytes = kSmallBN * kBKBytes;   // 16 KB of Wq per stage
constexpr int kBBytesPerKb = kSmallMP * kBKBytes;  // 2 KB of Xq per k-block
constexpr uint32_t kTmemCols = 32;
constexpr uint32_t kIdesc = idesc_i8_s32(kSmallBN, kSmallMP);

__device__ __forceinline__ int quantize_value(float x, float s) {
  const int q = __float2int_rn(__fdiv_rn(x, s));
  return max(-127, min(127, q));
}

__device__ __forceinline__ float habs_f(uint32_t word, int hi) {
  const unsigned short b = static_cast<unsigned short>(hi ? (word >> 16) : (word & 0xFFFFu));
  return fabsf(__half2float(__ushort_as_half(b)));
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

}  // namespace

// ------------------------------------------------------------------ stats

__global__ void __launch_bounds__(kThreads) small_stats_kernel(const SmallArgs a) {
  __shared__ __half2 red[8][32][4];
  __shared__ uint32_t flags[32];
  grid_dependency_wait();
  grid_launch_dependents();
  const int strip = blockIdx.x;
  const int chunk = threadIdx.x & 31;  // 8 columns each
  const int rg = threadIdx.x >> 5;     // rows rg and rg + 8
  const int col0 = strip * kStripCols + chunk * 8;
  const bool valid = col0 < a.K;
  uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
  if (valid && rg < a.M)
    v0 = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(rg) * a.K + col0));
  if (valid && rg + 8 < a.M)
    v1 = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(rg + 8) * a.K + col0));
  const uint32_t w0[4] = {v0.x, v0.y, v0.z, v0.w};
  const uint32_t w1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __half2 h0 = *reinterpret_cast<const __half2*>(&w0[e]);
    __half2 h1 = *reinterpret_cast<const __half2*>(&w1[e]);
    red[rg][chunk][e] = __hmax2(__habs2(h0), __habs2(h1));
  }
  __syncthreads();
  if (rg == 0) {
    uint32_t bits8 = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __half2 m = red[0][chunk][e];
#pragma unroll
      for (int r = 1; r < 8; ++r) m = __hmax2(m, red[r][chunk][e]);
      if (__low2float(m) > a.threshold) bits8 |= 1u << (2 * e);
      if (__high2float(m) > a.threshold) bits8 |= 1u << (2 * e + 1);
    }
    flags[chunk] = bits8;
    uint32_t word = bits8 << (8 * (chunk & 3));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    const int w = strip * (kStripCols / 32) + chunk / 4;
    if ((chunk & 3) == 0 && w < (a.K + 31) / 32) a.mask[w] = word;
  }
  __syncthreads();
  const uint32_t bits8 = flags[chunk];
  float r0 = 0.0f, r1 = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    if (!((bits8 >> e) & 1u)) {
      r0 = fmaxf(r0, habs_f(w0[e / 2], e & 1));
      r1 = fmaxf(r1, habs_f(w1[e / 2], e & 1));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    r0 = fmaxf(r0, __shfl_xor_sync(0xffffffffu, r0, o));
    r1 = fmaxf(r1, __shfl_xor_sync(0xffffffffu, r1, o));
  }
  if (chunk == 0) {
    a.rowmax_part[strip * kSmallMP + rg] = r0;
    a.rowmax_part[strip * kSmallMP + rg + 8] = r1;
  }
}

// ------------------------------------------------------------------ fused quantize + product

struct SmallShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t xq_ready;
  uint64_t tmem_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int last;
  int epi_ok;
  float sx[kSmallMP];
  int zero_row[kSmallMP];
  float psum[kSmallBN][kSmallMP + 1];  // this CTA's outlier term per channel (+1: no bank clash)
  uint32_t mask[kSmallMaxKbPerSplit * 4];
};

size_t small_gemm_smem_bytes(int kb_per_split) {
  return 1024 + static_cast<size_t>(kStages) * kABytes +
         static_cast<size_t>(kb_per_split) * kBBytesPerKb + sizeof(SmallShared);
}

__global__ void __launch_bounds__(kThreads, 2)
    small_gemm_kernel(const __grid_constant__ CUtensorMap map_wq, const SmallArgs a) {
  extern __shared__ uint8_t small_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(small_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a_stage = base;                                   // kStages x 16 KB
  uint8_t* xq_tiles = base + kStages * kABytes;              // nkb x 2 KB
  const int S = a.splits;
  const int tile = blockIdx.x / S, split = blockIdx.x % S;
  const int n0 = tile * kSmallBN;
  const int kb_total = (a.K + kBKBytes - 1) / kBKBytes;
  const int kb_begin = static_cast<int>(static_cast<long long>(split) * kb_total / S);
  const int kb_end = static_cast<int>(static_cast<long long>(split + 1) * kb_total / S);
  const int nkb = kb_end - kb_begin;
  SmallShared& sh = *reinterpret_cast<SmallShared*>(xq_tiles + nkb * kBBytesPerKb);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort = &sh.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    mbar_init(&sh.xq_ready, 192);
    mbar_init(&sh.tmem_full, 1);
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    sh.last = 0;
    fence_mbarrier_init();
  }
  if (threadIdx.x == 32) prefetch_tmap(&map_wq);
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ---- Wq stream: starts before the stats kernel has finished (weights are constant)
      bool ok = true;
      for (int j = 0; j < nkb; ++j) {
        const int s = j % kStages;
        if (j >= kStages &&
            !mbar_wait_bounded(&sh.empty[s], static_cast<uint32_t>((j / kStages) - 1) & 1u, abort)) {
          ok = false;
          int dummy = 0;
          for (int d = j - kStages; d < j; ++d)  // let the copies in flight land
            mbar_wait_bounded(&sh.full[d % kStages], static_cast<uint32_t>(d / kStages) & 1u,
                              &dummy);
          break;
        }
        mbar_arrive_expect_tx(&sh.full[s], kABytes);
        tma_load_2d(&map_wq, a_stage + s * kABytes, &sh.full[s], (kb_begin + j) * kBKBytes, n0);
      }
      if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
      if (ok) {  // let every copy land before the block may exit
        int dummy = 0;
        for (int d = nkb > kStages ? nkb - kStages : 0; d < nkb; ++d)
          mbar_wait_bounded(&sh.full[d % kStages], static_cast<uint32_t>(d / kStages) & 1u, &dummy);
      }
    }
  } else if (warp == 1) {
    grid_dependency_wait();
    if (lane == 0) {
      // ---- MMA issuer
      bool ok = mbar_wait_bounded(&sh.xq_ready, 0, abort);
      if (ok) {
        tc_fence_after();
        for (int j = 0; j < nkb; ++j) {
          const int s = j % kStages;
          if (!mbar_wait_bounded(&sh.full[s], static_cast<uint32_t>(j / kStages) & 1u, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_addr(a_stage + s * kABytes);
          const uint32_t b0 = smem_addr(xq_tiles + j * kBBytesPerKb);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8(tmem, sw128_kmajor_desc(a0 + 32u * k), sw128_kmajor_desc(b0 + 32u * k), kIdesc,
                   (j > 0 || k > 0) ? 1u : 0u);
          mma_commit(&sh.empty[s]);
        }
        if (ok) mma_commit(&sh.tmem_full);
      }
      mma_commit(&sh.drain);
      int dummy = 0;
      mbar_wait_bounded(&sh.drain, 0, &dummy);
      if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
    }
  } else {
    // ---- warps 2..7: quantize this CTA's K-slice of X into the B operand
    grid_dependency_wait();
    const int tq = threadIdx.x - 64;  // 0..191
    const int strips = (a.K + kStripCols - 1) / kStripCols;
    if (tq < kSmallMP) {
      float rm = 0.0f;
      for (int s = 0; s < strips; ++s) rm = fmaxf(rm, __ldcg(a.rowmax_part + s * kSmallMP + tq));
      sh.sx[tq] = (tq < a.M) ? __fdiv_rn(rm, 127.0f) : 0.0f;
      sh.zero_row[tq] = (tq >= a.M) || rm == 0.0f;
    }
    const int words = (a.K + 31) / 32;
    for (int w = tq; w < nkb * 4; w += 192) {
      const int gw = kb_begin * 4 + w;
      sh.mask[w] = gw < words ? __ldcg(a.mask + gw) : 0u;
    }
    named_barrier(1, 192);
    const int chunks_per_row = nkb * (kBKBytes / 8);  // 8 int8 codes per chunk
    for (int u = tq; u < kSmallMP * chunks_per_row; u += 192) {
      const int r = u / chunks_per_row, c = u % chunks_per_row;
      const int k = kb_begin * kBKBytes + c * 8;
      uint2 q = make_uint2(0u, 0u);
      if (r < a.M && k < a.K && !sh.zero_row[r]) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(r) * a.K + k));
        const uint32_t bits = (sh.mask[(c * 8) >> 5] >> ((c * 8) & 31)) & 0xFFu;
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        const float s = sh.sx[r];
        uint32_t p[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if ((bits >> e) & 1u) continue;
          const unsigned short hb = static_cast<unsigned short>((w[e / 2] >> (16 * (e & 1))) & 0xFFFFu);
          const int qv = quantize_value(__half2float(__ushort_as_half(hb)), s);
          p[e / 4] |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * (e & 3));
        }
        q = make_uint2(p[0], p[1]);
      }
      const int kbl = c / 16, kk = (c % 16) * 8;
      uint8_t* dst = xq_tiles + kbl * kBBytesPerKb + (r / 8) * 1024 + (r % 8) * 128 +
                     (((kk / 16) ^ (r % 8)) * 16) + (kk % 16);
      *reinterpret_cast<uint2*>(dst) = q;
    }
    fence_async_shared();
    mbar_arrive(&sh.xq_ready);

    if (warp >= 4) {
      // ---- warps 4..7 own TMEM lane quadrants 0..3, i.e. channels 32q .. 32q+31
      const int quad = warp & 3;
      const int n = quad * 32 + lane, gn = n0 + n;
      // The fp16 outlier term of the outlier columns inside this CTA's K-slice, computed
      // while the MMAs run: P[i] = sum_j X[i,j] * fp16(Wq[gn,j] * w_scale[gn]).
      {
        float P[kSmallMP];
#pragma unroll
        for (int i = 0; i < kSmallMP; ++i) P[i] = 0.0f;
        if (gn < a.N) {
          const float sw_n = a.w_scale[gn];
          const int8_t* wrow = a.Wq + static_cast<size_t>(gn) * a.K;
          for (int w = 0; w < nkb * 4; ++w) {
            uint32_t bits = sh.mask[w];
            while (bits) {
              const int j = kb_begin * kBKBytes + w * 32 + __ffs(bits) - 1;
              bits &= bits - 1u;
              const float wv = __half2float(__float2half_rn(static_cast<float>(wrow[j]) * sw_n));
#pragma unroll
              for (int i = 0; i < kSmallMP; ++i)
                if (i < a.M) P[i] += wv * __half2float(a.X[static_cast<size_t>(i) * a.K + j]);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < kSmallMP; ++i) sh.psum[n][i] = P[i];
      }
      int32_t acc[kSmallMP];
      mbar_wait_bounded(&sh.tmem_full, 0, abort);
      // one decision for all 128 epilogue threads, so the barriers below cannot split
      named_barrier(2, 128);
      if (threadIdx.x == 128) sh.epi_ok = (*abort == 0);
      named_barrier(2, 128);
      const bool ok = sh.epi_ok != 0;
      tc_fence_after();
      uint32_t r[16];
      __syncwarp();
      tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quad * 32) << 16), r);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) acc[i] = ok ? static_cast<int32_t>(r[i]) : 0;
      bool finish = ok;
      if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
      if (ok && S > 1) {
        const size_t slot = ((static_cast<size_t>(tile) * S + split) * kSmallBN + n) * kSmallMP;
        int4* ip = reinterpret_cast<int4*>(a.partials + slot);
        float4* fp = reinterpret_cast<float4*>(a.fpartials + slot);
#pragma unroll
        for (int v = 0; v < kSmallMP / 4; ++v) {
          __stcg(ip + v, make_int4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]));
          __stcg(fp + v, make_float4(sh.psum[n][4 * v], sh.psum[n][4 * v + 1],
                                     sh.psum[n][4 * v + 2], sh.psum[n][4 * v + 3]));
        }
        __threadfence();
        named_barrier(2, 128);
        if (threadIdx.x == 128) {
          const unsigned old = atomicAdd(a.counters + tile, 1u);
          const int last = old == static_cast<unsigned>(S - 1);
          if (last) atomicExch(a.counters + tile, 0u);  // ready for the next call
          sh.last = last;
        }
        named_barrier(2, 128);
        finish = sh.last != 0;
        if (finish) {
          __threadfence();
          float P[kSmallMP];
#pragma unroll
          for (int i = 0; i < kSmallMP; ++i) {
            acc[i] = 0;
            P[i] = 0.0f;
          }
          for (int s2 = 0; s2 < S; ++s2) {  // fixed order: the same bits on every call
            const size_t o = ((static_cast<size_t>(tile) * S + s2) * kSmallBN + n) * kSmallMP;
            const int4* ip2 = reinterpret_cast<const int4*>(a.partials + o);
            const float4* fp2 = reinterpret_cast<const float4*>(a.fpartials + o);
#pragma unroll
            for (int v = 0; v < kSmallMP / 4; ++v) {
              const int4 t = __ldcg(ip2 + v);
              const float4 f = __ldcg(fp2 + v);
              acc[4 * v] += t.x;
              acc[4 * v + 1] += t.y;
              acc[4 * v + 2] += t.z;
              acc[4 * v + 3] += t.w;
              P[4 * v] += f.x;
              P[4 * v + 1] += f.y;
              P[4 * v + 2] += f.z;
              P[4 * v + 3] += f.w;
            }
          }
#pragma unroll
          for (int i = 0; i < kSmallMP; ++i) sh.psum[n][i] = P[i];
        }
      }
      if (finish && gn < a.N) {
        const float b = a.bias ? __half2float(a.bias[gn]) : 0.0f;
        const float swn = a.w_scale[gn];
#pragma unroll
        for (int i = 0; i < kSmallMP; ++i) {
          if (i < a.M) {
            const float y = static_cast<float>(acc[i]) * sh.sx[i] * swn + sh.psum[n][i] + b;
            a.Y[static_cast<size_t>(i) * a.N + gn] = __float2half_rn(y);
            if (a.acc) a.acc[static_cast<size_t>(i) * a.N + gn] = acc[i];
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

SmallPlan plan_small(int M, int N, int K, int num_sms) {
  SmallPlan p;
  p.tiles = (N + kSmallBN - 1) / kSmallBN;
  const int kb_total = (K + kBKBytes - 1) / kBKBytes;
  int S = static_cast<int>((2.0 * num_sms) / p.tiles + 0.5);
  S = S < 1 ? 1 : S;
  const int need = (kb_total + kSmallMaxKbPerSplit - 1) / kSmallMaxKbPerSplit;
  if (S < need) S = need;
  if (S > kb_total) S = kb_total;
  if (S > kSmallMaxSplits) S = kSmallMaxSplits;
  p.splits = S;
  p.kb_per_split = (kb_total + S - 1) / S;
  p.strips = (K + kStripCols - 1) / kStripCols;
  (void)M;
  return p;
}

cudaError_t launch_small_stats(const SmallArgs& a, const SmallPlan& p, cudaStream_t stream,
                               bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.strips);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, small_stats_kernel, a);
}

cudaError_t launch_small_gemm(const CUtensorMap& map_wq, const SmallArgs& a, const SmallPlan& p,
                              cudaStream_t stream, bool pdl) {
  const size_t smem = small_gemm_smem_bytes(p.kb_per_split);
  static size_t configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(small_gemm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(small_gemm_smem_bytes(kSmallMaxKbPerSplit)));
    if (e != cudaSuccess) return e;
    configured = small_gemm_smem_bytes(kSmallMaxKbPerSplit);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.tiles * p.splits);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, small_gemm_kernel, map_wq, a);
}

}  // namespace i8mm
