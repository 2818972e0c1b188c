// gemv.cu -- the LLM.int8() layer for a few tokens (M <= 16), the weight-streaming regime.
//
// With M <= 16 the layer reads every byte of Wq once and does M multiply-adds per byte:
// it is bound by HBM, not by the tensor cores (a tcgen05 MMA with M = 128 channels costs
// the same time at N = 16 tokens as at N = 256, so it would run at 1/16 of its rate).
// This kernel therefore streams Wq at full bandwidth and multiplies on the CUDA cores:
//
//   * one CTA per SM owns C <= 32 output channels over all of K (no split-K, no reduction
//     across CTAs); its first instruction starts the TMA stream of its Wq rows into a
//     shared-memory ring (all of it when it fits);
//   * meanwhile its 512 threads read X (M x K, from L2 after the first CTA) and find the
//     outlier columns, max_i |x| > threshold ([P2] "8位量化实战：离群值处理与显存优化避坑
//     指南" section 2.3), the row scales sx = max over the regular columns / 127 and the
//     int8 codes q = rne(x / sx) clamped to [-127, 127], 0 in outlier columns ([P5]
//     "PyTorch 2.9 支持 LLM.int8()" item 2); every CTA does this redundantly, which costs
//     less than any exchange between CTAs;
//   * acc[i,n] = sum_k q[i,k] * Wq[n,k] exactly in int32 with dp4a, lanes splitting each
//     256-byte slab of K and a warp reduction at the end;
//   * the fp16 outlier term sum_{j in O} X[i,j] * fp16(Wq[n,j] * w_scale[n]) ([P5] "如何在
//     PyTorch 2.9 中启用 LLM.int8 推理": no fp16 weights are kept) and the epilogue
//     Y = fp16(acc * sx * w_scale + P + bias) follow in the same warps.
//
// Quantization arithmetic, exact to the IEEE quotient: v = x * r with r = 1/sx rounded to
// nearest is within 2^-16 of x/sx (|x/sx| <= 127) and the rounded quotient fl(x/sx) is
// within 2^-18 of x/sx, so rne(v) = rne(fl(x/sx)) unless v lies within 2^-15 of a
// half-integer; there the quotient itself (__fdiv_rn) is rounded.
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSlab = 256;              // bytes of K per ring stage (and per TMA box row)
constexpr int kMaxChannels = 32;        // per CTA
constexpr int kChPerWarp = kMaxChannels / kWarps;  // 2
constexpr int kMaxStages = 64;
constexpr size_t kSmemLimit = 227 * 1024;

__device__ __forceinline__ float h2f(uint32_t word, int hi) {
  return __half2float(
      __ushort_as_half(static_cast<unsigned short>(hi ? (word >> 16) : (word & 0xFFFFu))));
}

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// 8 codes of one row chunk, packed little-endian (see the file comment for exactness)
__device__ __forceinline__ uint2 quantize8(const uint4& v, float sc, float rcp, uint32_t bits) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float x[8];
  int qv[8];
  uint32_t near_tie = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    x[e] = h2f(w[e / 2], e & 1);
    const float t = x[e] * rcp;
    qv[e] = __float2int_rn(t);
    const float d = fabsf(t - rintf(t));
    near_tie |= (fabsf(d - 0.5f) <= 0x1p-15f ? 1u : 0u) << e;
  }
  if (near_tie) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if ((near_tie >> e) & 1u) qv[e] = __float2int_rn(__fdiv_rn(x[e], sc));
  }
  uint32_t p[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int qc = max(-127, min(127, qv[e]));
    const uint32_t code = ((bits >> e) & 1u) ? 0u : (static_cast<uint32_t>(qc) & 0xFFu);
    p[e / 4] |= code << (8 * (e & 3));
  }
  return make_uint2(p[0], p[1]);
}

}  // namespace

struct GemvShared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  float red[kWarps][kSmallMP];
  float sx[kSmallMP];
  float rcp[kSmallMP];
  int zero_row[kSmallMP];
  int abort;
};

// [Wq ring: stages x C x 256 B | Xq: MT x kpad | flags: kpad/8 | GemvShared]
size_t gemv_smem_bytes(int stages, int C, int MT, int kpad) {
  return 1024 + static_cast<size_t>(stages) * C * kSlab + static_cast<size_t>(MT) * kpad +
         kpad / 8 + sizeof(GemvShared) + 16;
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap map_wq, const GemvArgs a) {
  extern __shared__ uint8_t gemv_smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gemv_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int C = a.channels, R = a.stages, kpad = a.kpad;
  const int nst = kpad / kSlab;  // ring stages to consume
  const int stage_bytes = C * kSlab;
  int8_t* xq = reinterpret_cast<int8_t*>(ring + static_cast<size_t>(R) * stage_bytes);
  uint8_t* flags = reinterpret_cast<uint8_t*>(xq + static_cast<size_t>(MT) * kpad);
  GemvShared& sh = *reinterpret_cast<GemvShared*>(
      (reinterpret_cast<uintptr_t>(flags + kpad / 8) + 15) & ~static_cast<uintptr_t>(15));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * C;
  const int M = a.M, K = a.K;
  volatile int* abort = &sh.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], kWarps);
    }
    sh.abort = 0;
    fence_mbarrier_init();
    prefetch_tmap(&map_wq);
  }
  __syncthreads();
  grid_dependency_wait();  // the inputs may come from the previous launch on the stream

  if (threadIdx.x == 0) {  // start the weight stream before touching X
    const int first = nst < R ? nst : R;
    for (int j = 0; j < first; ++j) {
      mbar_arrive_expect_tx(&sh.full[j], stage_bytes);
      tma_load_2d(&map_wq, ring + static_cast<size_t>(j) * stage_bytes, &sh.full[j], j * kSlab, n0);
    }
  }

  // ---- pass 1: outlier columns and row maxima over the regular columns
  const int chunks = kpad / 8;  // 8-column chunks, K padded to the slab
  float rmax[MT];
#pragma unroll
  for (int i = 0; i < MT; ++i) rmax[i] = 0.0f;
  for (int c = threadIdx.x; c < chunks; c += kThreads) {
    const int k = c * 8;
    uint4 v[MT];
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      v[i] = make_uint4(0u, 0u, 0u, 0u);
      if (i < M && k < K)
        v[i] = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * K + k));
    }
    __half2 cm[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) cm[e] = __float2half2_rn(0.0f);
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        cm[e] = __hmax2(cm[e], __habs2(*reinterpret_cast<const __half2*>(&w[e])));
    }
    uint32_t bits = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (__low2float(cm[e]) > a.threshold) bits |= 1u << (2 * e);
      if (__high2float(cm[e]) > a.threshold) bits |= 1u << (2 * e + 1);
    }
    flags[c] = static_cast<uint8_t>(bits);
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (!((bits >> e) & 1u)) rmax[i] = fmaxf(rmax[i], fabsf(h2f(w[e / 2], e & 1)));
    }
  }
#pragma unroll
  for (int i = 0; i < MT; ++i) {
    float m = rmax[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) sh.red[warp][i] = m;
  }
  __syncthreads();
  if (threadIdx.x < MT) {
    const int i = threadIdx.x;
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, sh.red[w][i]);
    const float sc = __fdiv_rn(m, 127.0f);
    sh.sx[i] = (i < M) ? sc : 0.0f;
    sh.rcp[i] = (i < M && m > 0.0f) ? __frcp_rn(sc) : 0.0f;
    sh.zero_row[i] = (i >= M) || m == 0.0f;
  }
  __syncthreads();

  // ---- pass 2: int8 activations into shared memory, xq[i * kpad + k] (X re-read from L1/L2)
  for (int c = threadIdx.x; c < chunks; c += kThreads) {
    const int k = c * 8;
    const uint32_t bits = flags[c];
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      uint2 q = make_uint2(0u, 0u);
      if (!sh.zero_row[i] && k < K) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * K + k));
        q = quantize8(v, sh.sx[i], sh.rcp[i], bits);
      }
      *reinterpret_cast<uint2*>(xq + static_cast<size_t>(i) * kpad + k) = q;
    }
  }
  __syncthreads();

  // ---- int32 products on the CUDA cores: warp w owns channels w and w + 16 of the CTA;
  // lane l owns bytes [8l, 8l + 8) of every 256-byte slab of K.
  int ch_count = a.N - n0;
  if (ch_count > C) ch_count = C;
  int32_t acc[kChPerWarp][MT];
#pragma unroll
  for (int r = 0; r < kChPerWarp; ++r)
#pragma unroll
    for (int i = 0; i < MT; ++i) acc[r][i] = 0;
  bool ok = true;
  for (int j = 0; j < nst; ++j) {
    const int s = j % R;
    const bool landed = mbar_wait_bounded(&sh.full[s], static_cast<uint32_t>(j / R) & 1u, abort);
    if (!__all_sync(0xffffffffu, landed)) {  // a warp-uniform decision
      ok = false;
      break;
    }
    const uint8_t* tile = ring + static_cast<size_t>(s) * stage_bytes;
    uint2 xw[MT];
#pragma unroll
    for (int i = 0; i < MT; ++i)
      xw[i] = (i < M) ? *reinterpret_cast<const uint2*>(xq + static_cast<size_t>(i) * kpad +
                                                       j * kSlab + 8 * lane)
                      : make_uint2(0u, 0u);
#pragma unroll
    for (int r = 0; r < kChPerWarp; ++r) {
      const int ch = warp + kWarps * r;
      if (ch < ch_count) {
        const uint2 ww = *reinterpret_cast<const uint2*>(tile + ch * kSlab + 8 * lane);
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          acc[r][i] = __dp4a(static_cast<int>(ww.x), static_cast<int>(xw[i].x), acc[r][i]);
          acc[r][i] = __dp4a(static_cast<int>(ww.y), static_cast<int>(xw[i].y), acc[r][i]);
        }
      }
    }
    if (j + R < nst) {  // refill this stage once every warp is done with it
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.empty[s]);
      if (threadIdx.x == 0) {
        if (!mbar_wait_bounded(&sh.empty[s], static_cast<uint32_t>(j / R) & 1u, abort)) {
          ok = false;
        } else {
          mbar_arrive_expect_tx(&sh.full[s], stage_bytes);
          tma_load_2d(&map_wq, ring + static_cast<size_t>(s) * stage_bytes, &sh.full[s],
                      (j + R) * kSlab, n0);
        }
      }
    }
  }
  if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);

  // ---- fp16 outlier term: lanes stride over the outlier flags; weight bytes come from the
  // resident ring when the whole slice fits, from global memory otherwise
  float P[kChPerWarp][MT];
#pragma unroll
  for (int r = 0; r < kChPerWarp; ++r)
#pragma unroll
    for (int i = 0; i < MT; ++i) P[r][i] = 0.0f;
  const bool resident = nst <= R;
  for (int c = lane; c < chunks; c += 32) {
    uint32_t bits = flags[c];
    while (bits) {
      const int j = c * 8 + __ffs(bits) - 1;
      bits &= bits - 1u;
      float xv[MT];
#pragma unroll
      for (int i = 0; i < MT; ++i)
        xv[i] = (i < M) ? __half2float(a.X[static_cast<size_t>(i) * K + j]) : 0.0f;
#pragma unroll
      for (int r = 0; r < kChPerWarp; ++r) {
        const int ch = warp + kWarps * r;
        if (ch < ch_count) {
          const int8_t q = resident ? static_cast<int8_t>(ring[static_cast<size_t>(j / kSlab) * stage_bytes +
                                                              ch * kSlab + j % kSlab])
                                    : a.Wq[static_cast<size_t>(n0 + ch) * K + j];
          const float wv = __half2float(__float2half_rn(static_cast<float>(q) * a.w_scale[n0 + ch]));
#pragma unroll
          for (int i = 0; i < MT; ++i) P[r][i] += wv * xv[i];
        }
      }
    }
  }

  // ---- reduce over the 32 lanes and write Y (lane l writes pair (r, i) = (l / MT, l % MT))
#pragma unroll
  for (int r = 0; r < kChPerWarp; ++r) {
#pragma unroll
    for (int i = 0; i < MT; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        acc[r][i] += __shfl_xor_sync(0xffffffffu, acc[r][i], o);
        P[r][i] += __shfl_xor_sync(0xffffffffu, P[r][i], o);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kChPerWarp; ++r) {
    const int ch = warp + kWarps * r;
    const int n = n0 + ch;
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      if (lane == (r * MT + i) % 32 && ch < ch_count && i < M) {
        const float b = a.bias ? __half2float(a.bias[n]) : 0.0f;
        const float y = static_cast<float>(acc[r][i]) * sh.sx[i] * a.w_scale[n] + P[r][i] + b;
        a.Y[static_cast<size_t>(i) * a.N + n] = __float2half_rn(y);
        if (a.acc) a.acc[static_cast<size_t>(i) * a.N + n] = ok ? acc[r][i] : 0;
      }
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ host side

GemvPlan plan_gemv(int M, int N, int K, int num_sms) {
  GemvPlan p;
  p.mt = M <= 8 ? 8 : kSmallMP;
  int C = (N + num_sms - 1) / num_sms;
  if (C < 1) C = 1;
  if (C > kMaxChannels) C = kMaxChannels;
  p.channels = C;
  p.ctas = (N + C - 1) / C;
  p.kpad = (K + kSlab - 1) / kSlab * kSlab;
  const int nst = p.kpad / kSlab;
  int R = nst < kMaxStages ? nst : kMaxStages;
  while (R > 2 && gemv_smem_bytes(R, C, p.mt, p.kpad) > kSmemLimit) --R;
  p.stages = R;
  p.fits = M <= kSmallMP && gemv_smem_bytes(R, C, p.mt, p.kpad) <= kSmemLimit;
  return p;
}

cudaError_t launch_gemv(const CUtensorMap& map_wq, const GemvArgs& a, const GemvPlan& p,
                        cudaStream_t stream, bool pdl) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != configured_device) {
    e = cudaFuncSetAttribute(gemv_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemLimit));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemv_kernel<kSmallMP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSmemLimit));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = gemv_smem_bytes(p.stages, p.channels, p.mt, p.kpad);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return p.mt == 8 ? cudaLaunchKernelEx(&cfg, gemv_kernel<8>, map_wq, a)
                   : cudaLaunchKernelEx(&cfg, gemv_kernel<kSmallMP>, map_wq, a);
}

}  // namespace i8mm
