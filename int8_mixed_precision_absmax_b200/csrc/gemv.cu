// gemv.cu -- the LLM.int8() layer for a few tokens (M <= 16), the weight-streaming regime.
//
// With M <= 16 the layer reads every byte of Wq once and does M multiply-adds per byte:
// it is bound by HBM, not by the tensor cores (a tcgen05 MMA with M = 128 channels costs
// the same time at N = 16 tokens as at N = 256, so it would run at 1/16 of its rate).
// Two launches:
//
//   few_quant_kernel  one thread-block cluster (<= 8 CTAs, each a strip of columns) reads X
//                     once and finds the outlier columns, max_i |x| > threshold ([P2]
//                     "8位量化实战：离群值处理与显存优化避坑指南" section 2.3), the row scales
//                     sx = max over the regular columns / 127 -- the strips exchange their
//                     row maxima and outlier counts through distributed shared memory --
//                     and writes q = rne(x / sx) clamped to [-127, 127], 0 in outlier
//                     columns ([P5] "PyTorch 2.9 支持 LLM.int8()" item 2), as int8 rows
//                     padded to 16, plus the compact outlier list with its fp16 values.
//   gemv_kernel       each CTA owns 32 output channels over all of K (no split-K, no
//                     reduction across CTAs).  It starts the TMA stream of its Wq rows into
//                     shared memory (32 KB boxes: 32 rows x 8 swizzled 128-byte k-blocks)
//                     before it waits for the quantization (that kernel lets it start only
//                     after its own inputs were complete; the weights are not written by it).
//                     Each warp owns a range of K and computes acc[i,n] = sum_k q[i,k]*Wq[n,k]
//                     exactly with the int8 warp-level MMA m16n8k32 (16 channels x 8 tokens x
//                     32 K per instruction; a tcgen05 MMA with M = 128 channels takes the same
//                     time at N = 8 tokens as at N = 256, so at this shape it would idle);
//                     the warps' partial sums meet in shared memory.  The fp16 outlier term
//                     sum_{j in O} X[i,j] * fp16(Wq[n,j] * w_scale[n]) ([P5] "如何在 PyTorch
//                     2.9 中启用 LLM.int8 推理": no fp16 weights are kept) comes from the
//                     compact list, and Y = fp16(acc * sx * w_scale + P + bias).
//
// Quantization arithmetic: the codes of the IEEE quotient x / sx (codes.cuh).
#include "codes.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kSlab = 256;              // activation rows are padded to this many bytes
constexpr size_t kSmemLimit = 227 * 1024;
constexpr int kQThreads = 256;          // per CTA of the quantization cluster
constexpr int kQMaxCtas = 8;            // portable cluster size
constexpr int kGThreads = 512;          // per CTA of the product
constexpr int kGWarps = kGThreads / 32;
constexpr int kCh = 32;                 // output channels per CTA: two m16 tiles
constexpr int kBoxKb = 8;               // 128-byte k-blocks per TMA box
constexpr int kBoxBytes = kCh * kBoxKb * 128;  // 32 KB
constexpr int kMaxBoxes = 6;            // ring depth (boxes)

__device__ __forceinline__ float h2f(uint32_t word, int hi) {
  return __half2float(
      __ushort_as_half(static_cast<unsigned short>(hi ? (word >> 16) : (word & 0xFFFFu))));
}

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// 8 codes of one row chunk, packed little-endian, outlier columns (bits) 0 (codes.cuh)
__device__ __forceinline__ uint2 quantize8(const uint4& v, float sc, float rcp, uint32_t bits) {
  const uint2 q = codes8(v, sc, rcp);
  const uint2 keep = keep_bytes(bits);
  return make_uint2(q.x & keep.x, q.y & keep.y);
}

// D(16 x 8, int32) += A(16 x 32, int8, row-major) * B(32 x 8, int8, column-major)
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

}  // namespace

// ------------------------------------------------------------------ activation quantization

constexpr int kQMaxChunks = 256;  // chunks per CTA of the cluster: strip of 2048 columns

struct FewQuantShared {
  uint8_t flags[kQMaxChunks];    // outlier bits of this strip's chunks
  int chunk_pos[kQMaxChunks];    // position of a chunk's first outlier in the list
  float red[kQThreads / 32][kSmallMP];
  float rowmax_local[kSmallMP];  // read by the other CTAs of the cluster
  int count_local;               // read by the other CTAs of the cluster
  int warp_count[kQThreads / 32];
  float sx[kSmallMP];
  float rcp[kSmallMP];
  int zero_row[kSmallMP];
  int base;
};

template <int MT>
__global__ void __launch_bounds__(kQThreads) few_quant_kernel(const GemvArgs a) {
  __shared__ FewQuantShared sh;
  // Everything this kernel reads may come from the previous launch; once that is complete,
  // the product kernel may start its weight stream.
  grid_dependency_wait();
  grid_launch_dependents();
  const int Q = static_cast<int>(gridDim.x);
  const int r = static_cast<int>(cluster_rank());
  const int chunks = a.kpad / 8;
  const int c_begin = static_cast<int>(static_cast<long long>(r) * chunks / Q);
  const int c_end = static_cast<int>(static_cast<long long>(r + 1) * chunks / Q);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int M = a.M, K = a.K;
  // thread t owns the contiguous chunks [t_begin, t_end) of this strip, so the outlier list
  // comes out in ascending column order
  const int per = (c_end - c_begin + kQThreads - 1) / kQThreads;
  const int t_begin = min(c_end, c_begin + static_cast<int>(threadIdx.x) * per);
  const int t_end = min(c_end, t_begin + per);
  const bool one_chunk = per <= 1;

  // ---- phase 1: outlier flags and row maxima of this strip
  float rmax[MT];
#pragma unroll
  for (int i = 0; i < MT; ++i) rmax[i] = 0.0f;
  uint4 v[MT];
  uint32_t my_bits = 0;
  int my_count = 0;
  auto load_chunk = [&](int c) {
    const int k = c * 8;
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      v[i] = make_uint4(0u, 0u, 0u, 0u);
      if (i < M && k < K)
        v[i] = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * K + k));
    }
  };
  auto chunk_flags = [&]() {
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
    return bits;
  };
  for (int c = t_begin; c < t_end; ++c) {
    load_chunk(c);
    const uint32_t bits = chunk_flags();
    my_count += __popc(bits);
    if (one_chunk) my_bits = bits;
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (!((bits >> e) & 1u)) rmax[i] = fmaxf(rmax[i], fabsf(h2f(w[e / 2], e & 1)));
    }
  }
  // row maxima over the strip and the strip's outlier count (exclusive scan per thread)
#pragma unroll
  for (int i = 0; i < MT; ++i) {
    float m = rmax[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) sh.red[warp][i] = m;
  }
  int incl = my_count;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh.warp_count[warp] = incl;
  __syncthreads();
  int my_off = incl - my_count;
  for (int w = 0; w < warp; ++w) my_off += sh.warp_count[w];
  if (threadIdx.x < MT) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kQThreads / 32; ++w) m = fmaxf(m, sh.red[w][threadIdx.x]);
    sh.rowmax_local[threadIdx.x] = m;
  }
  if (threadIdx.x == 0) {
    int total = 0;
    for (int w = 0; w < kQThreads / 32; ++w) total += sh.warp_count[w];
    sh.count_local = total;
  }
  cluster_sync_all();  // every strip's maxima and count are in its shared memory

  // ---- the row scales over all strips, and this strip's place in the outlier list
  if (threadIdx.x < MT) {
    const int i = threadIdx.x;
    const uint32_t local = smem_addr(&sh.rowmax_local[i]);
    float m = 0.0f;
    for (int q = 0; q < Q; ++q) m = fmaxf(m, ld_cluster_f32(map_rank(local, q)));
    if (a.per_tensor)  // one scale for all rows: the largest row absmax (rows past M hold 0)
#pragma unroll
      for (int o = 1; o < MT; o <<= 1) m = fmaxf(m, __shfl_xor_sync((1u << MT) - 1u, m, o));
    const float sc = __fdiv_rn(m, 127.0f);
    sh.sx[i] = (i < M) ? sc : 0.0f;
    sh.rcp[i] = (i < M && m > 0.0f) ? __frcp_rn(sc) : 0.0f;
    sh.zero_row[i] = (i >= M) || m == 0.0f;
    if (r == 0) a.sx[i] = sh.sx[i];
  }
  if (threadIdx.x == 32) {
    const uint32_t local = smem_addr(&sh.count_local);
    int base = 0, total = 0;
    for (int q = 0; q < Q; ++q) {
      const int cq = ld_cluster_s32(map_rank(local, q));
      if (q < r) base += cq;
      total += cq;
    }
    sh.base = base;
    if (r == 0) *a.n_out = total;
  }
  __syncthreads();

  // ---- phase 2: int8 rows xq[i * kpad + k] over (row, chunk) units, and the compact
  // outlier list (chunk c's outliers start at chunk_pos[c])
  if (one_chunk && t_begin < t_end) {
    sh.flags[t_begin - c_begin] = static_cast<uint8_t>(my_bits);
    sh.chunk_pos[t_begin - c_begin] = sh.base + my_off;
  }
  __syncthreads();
  const int nch = c_end - c_begin;
  if (one_chunk) {
    for (int u = threadIdx.x; u < MT * nch; u += kQThreads) {
      const int i = u / nch, cl = u % nch;
      const int k = (c_begin + cl) * 8;
      uint2 q = make_uint2(0u, 0u);
      if (!sh.zero_row[i] && k < K) {
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * K + k));
        q = quantize8(x, sh.sx[i], sh.rcp[i], sh.flags[cl]);
      }
      *reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(i) * a.kpad + k) = q;
    }
    for (int cl = threadIdx.x; cl < nch; cl += kQThreads) {
      uint32_t b = sh.flags[cl];
      int pos = sh.chunk_pos[cl];
      const int k = (c_begin + cl) * 8;
      while (b) {
        const int e = __ffs(b) - 1;
        b &= b - 1u;
        a.cols[pos] = k + e;
        for (int i = 0; i < kSmallMP; ++i)
          a.xo[static_cast<size_t>(pos) * kSmallMP + i] =
              (i < M) ? a.X[static_cast<size_t>(i) * K + k + e] : __float2half_rn(0.0f);
        ++pos;
      }
    }
  } else {
    int pos = sh.base + my_off;
    for (int c = t_begin; c < t_end; ++c) {
      load_chunk(c);
      const uint32_t bits = chunk_flags();
      const int k = c * 8;
#pragma unroll
      for (int i = 0; i < MT; ++i) {
        uint2 q = make_uint2(0u, 0u);
        if (!sh.zero_row[i] && k < K) q = quantize8(v[i], sh.sx[i], sh.rcp[i], bits);
        *reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(i) * a.kpad + k) = q;
      }
      uint32_t b = bits;
      while (b) {
        const int e = __ffs(b) - 1;
        b &= b - 1u;
        a.cols[pos] = k + e;
        for (int i = 0; i < kSmallMP; ++i)
          a.xo[static_cast<size_t>(pos) * kSmallMP + i] =
              (i < M) ? a.X[static_cast<size_t>(i) * K + k + e] : __float2half_rn(0.0f);
        ++pos;
      }
    }
  }
  cluster_sync_all();  // no CTA leaves while the others may still read its shared memory
}

// ------------------------------------------------------------------ product

constexpr int kMaxStagedOutliers = 256;  // outlier columns staged in shared memory

struct GemvShared {
  uint64_t full[kMaxBoxes];
  uint64_t empty[kMaxBoxes];
  float sx[kSmallMP];
  float wscale[kCh];
  float bias[kCh];
  int cols[kMaxStagedOutliers];
  __half xo[kMaxStagedOutliers][kSmallMP];
  int n_out;
  int abort;
  int issued;  // boxes whose copy was started
};

// [Wq ring: boxes x 32 KB | partial sums: 16 warps x 32 channels x MT | GemvShared]
size_t gemv_smem_bytes(int boxes, int MT) {
  return 1024 + static_cast<size_t>(boxes) * kBoxBytes +
         static_cast<size_t>(kGWarps) * kCh * MT * sizeof(int32_t) + sizeof(GemvShared) + 16;
}

// byte (row, kk) of a 32-row tile of 128-byte rows written with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128_offset(int row, int kk) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 +
                               ((((kk >> 4) ^ (row & 7))) << 4) + (kk & 15));
}

template <int MT>
__global__ void __launch_bounds__(kGThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap map_wq, const GemvArgs a) {
  extern __shared__ uint8_t gemv_smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gemv_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int R = a.stages;                       // ring depth in boxes
  const int kb_total = a.K / 128;               // 128-byte k-blocks (K % 128 == 0 here)
  const int nbox = (kb_total + kBoxKb - 1) / kBoxKb;
  int32_t* red = reinterpret_cast<int32_t*>(ring + static_cast<size_t>(R) * kBoxBytes);
  GemvShared& sh = *reinterpret_cast<GemvShared*>(red + kGWarps * kCh * MT);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * kCh;
  const int M = a.M;
  volatile int* abort = &sh.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], kGWarps);
    }
    sh.abort = 0;
    fence_mbarrier_init();
    prefetch_tmap(&map_wq);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // the weight stream starts before the activations are ready
    const int first = nbox < R ? nbox : R;
    for (int b = 0; b < first; ++b) {
      mbar_arrive_expect_tx(&sh.full[b], kBoxBytes);
      tma_load_3d(&map_wq, ring + static_cast<size_t>(b) * kBoxBytes, &sh.full[b], 0, n0,
                  b * kBoxKb);
    }
    sh.issued = first;
  }
  grid_dependency_wait();  // the quantization kernel is complete from here on

  // ---- this warp's k32 steps: [s_begin, s_end) of K/32, inside one box each time
  const int steps = a.K / 32;
  const int per = (steps + kGWarps - 1) / kGWarps;
  const int s_begin = min(steps, warp * per), s_end = min(steps, s_begin + per);
  const int g = lane >> 2, tig = lane & 3;
  constexpr int NT = MT / 8;  // n8 tiles of tokens
  int d[2][NT][4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[m][t][e] = 0;
  // all of this warp's int8-X fragments in one batch of loads (L2), before any wait
  constexpr int kMaxSteps = 16;  // k32 steps per warp: K <= 16 warps x 16 x 32 = 8192
  uint32_t bfr[kMaxSteps][NT][2];
#pragma unroll
  for (int u = 0; u < kMaxSteps; ++u)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      bfr[u][t][0] = bfr[u][t][1] = 0u;
      if (s_begin + u < s_end) {
        const int8_t* xrow = a.xq + static_cast<size_t>(t * 8 + g) * a.kpad + (s_begin + u) * 32 + 4 * tig;
        bfr[u][t][0] = __ldcg(reinterpret_cast<const unsigned int*>(xrow));
        bfr[u][t][1] = __ldcg(reinterpret_cast<const unsigned int*>(xrow + 16));
      }
    }
  bool ok = true;
  int waited_box = -1;
#pragma unroll
  for (int u = 0; u < kMaxSteps; ++u) {
    const int st = s_begin + u;
    if (st >= s_end) break;
    const int k0 = st * 32;
    const int box = k0 / (kBoxKb * 128);
    if (box != waited_box) {  // boxes are consumed in order; R >= boxes here (resident)
      const int slot = box % R;
      const uint32_t parity = static_cast<uint32_t>(box / R) & 1u;
      bool landed = true;
      if (lane == 0) landed = mbar_wait_bounded(&sh.full[slot], parity, abort);
      if (!__shfl_sync(0xffffffffu, landed ? 1 : 0, 0)) {
        ok = false;
        break;
      }
      mbar_try_wait(&sh.full[slot], parity);  // each lane observes the completed phase
      waited_box = box;
    }
    const uint8_t* tile = ring + static_cast<size_t>(box % R) * kBoxBytes +
                          ((k0 / 128) % kBoxKb) * (kCh * 128);
    const int kk = k0 % 128 + 4 * tig;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      uint32_t af[4];
      af[0] = *reinterpret_cast<const uint32_t*>(tile + sw128_offset(m * 16 + g, kk));
      af[1] = *reinterpret_cast<const uint32_t*>(tile + sw128_offset(m * 16 + g + 8, kk));
      af[2] = *reinterpret_cast<const uint32_t*>(tile + sw128_offset(m * 16 + g, kk + 16));
      af[3] = *reinterpret_cast<const uint32_t*>(tile + sw128_offset(m * 16 + g + 8, kk + 16));
#pragma unroll
      for (int t = 0; t < NT; ++t) mma_s8_16832(d[m][t], af, bfr[u][t][0], bfr[u][t][1]);
    }
  }
  if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
  // partial sums to shared memory: red[warp][channel][token]
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      int32_t* rw = red + static_cast<size_t>(warp) * kCh * MT;
      rw[(m * 16 + g) * MT + t * 8 + 2 * tig] = d[m][t][0];
      rw[(m * 16 + g) * MT + t * 8 + 2 * tig + 1] = d[m][t][1];
      rw[(m * 16 + g + 8) * MT + t * 8 + 2 * tig] = d[m][t][2];
      rw[(m * 16 + g + 8) * MT + t * 8 + 2 * tig + 1] = d[m][t][3];
    }
  if (threadIdx.x < kSmallMP) sh.sx[threadIdx.x] = __ldcg(a.sx + threadIdx.x);
  if (threadIdx.x < kCh) {
    const int n = n0 + threadIdx.x;
    sh.wscale[threadIdx.x] = n < a.N ? a.w_scale[n] : 0.0f;
    sh.bias[threadIdx.x] = (a.bias && n < a.N) ? __half2float(a.bias[n]) : 0.0f;
  }
  const int n_out = __ldcg(a.n_out);
  const int staged = n_out < kMaxStagedOutliers ? n_out : kMaxStagedOutliers;
  for (int t = threadIdx.x; t < staged * (kSmallMP + 1); t += kGThreads) {
    const int o = t / (kSmallMP + 1), i = t % (kSmallMP + 1);
    if (i == kSmallMP) sh.cols[o] = __ldcg(a.cols + o);
    else sh.xo[o][i] = a.xo[static_cast<size_t>(o) * kSmallMP + i];
  }
  __syncthreads();

  // ---- thread (c, i): sum the warps, add the outlier term and bias, write Y[i, n0 + c]
  const bool resident = nbox <= R;
  for (int t = threadIdx.x; t < kCh * MT; t += kGThreads) {
    const int c = t % kCh, i = t / kCh, n = n0 + c;
    if (i >= M || n >= a.N) continue;
    int32_t acc = 0;
#pragma unroll
    for (int w = 0; w < kGWarps; ++w) acc += red[(static_cast<size_t>(w) * kCh + c) * MT + i];
    const float swn = sh.wscale[c];
    float P = 0.0f;
    for (int o = 0; o < n_out; ++o) {
      const int j = o < staged ? sh.cols[o] : __ldcg(a.cols + o);
      float wv;
      if (a.W16) {
        wv = __half2float(a.W16[static_cast<size_t>(n) * a.K + j]);
      } else {
        int8_t q;
        if (resident) {
          const int kb = j / 128;
          const uint8_t* tile = ring + static_cast<size_t>(kb / kBoxKb) * kBoxBytes +
                                (kb % kBoxKb) * (kCh * 128);
          q = static_cast<int8_t>(tile[sw128_offset(c, j % 128)]);
        } else {
          q = a.Wq[static_cast<size_t>(n) * a.K + j];
        }
        wv = __half2float(__float2half_rn(static_cast<float>(q) * swn));
      }
      if (i == 0 && a.trace.what) a.trace.what[static_cast<size_t>(n) * a.K + j] = __float2half_rn(wv);
      P += wv * __half2float(o < staged ? sh.xo[o][i] : a.xo[static_cast<size_t>(o) * kSmallMP + i]);
    }
    const float bb = sh.bias[c];
    const float y = static_cast<float>(acc) * sh.sx[i] * swn + P + bb;
    a.Y[static_cast<size_t>(i) * a.N + n] = __float2half_rn(y);
    if (a.acc) a.acc[static_cast<size_t>(i) * a.N + n] = ok ? acc : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0 && sh.abort) {
    // a wait gave up: let the copies still in flight land before the block exits
    int dummy = 0;
    for (int b2 = sh.issued > R ? sh.issued - R : 0; b2 < sh.issued; ++b2)
      mbar_wait_bounded(&sh.full[b2 % R], static_cast<uint32_t>(b2 / R) & 1u, &dummy);
  }
}

// ------------------------------------------------------------------ host side

GemvPlan plan_gemv(int M, int N, int K, int num_sms) {
  (void)num_sms;
  GemvPlan p;
  p.mt = M <= 8 ? 8 : kSmallMP;
  p.channels = kCh;
  p.ctas = (N + kCh - 1) / kCh;
  p.kpad = (K + kSlab - 1) / kSlab * kSlab;
  const int nbox = (K / 128 + kBoxKb - 1) / kBoxKb;
  p.stages = nbox;  // the whole slice stays resident: the outlier term reads it back
  const int chunks = p.kpad / 8;
  int Q = (chunks + 63) / 64;  // about 64 chunks (512 columns) per CTA of the cluster
  p.quant_ctas = Q < 1 ? 1 : (Q > kQMaxCtas ? kQMaxCtas : Q);
  const int chunks_per_cta = (chunks + p.quant_ctas - 1) / p.quant_ctas;
  p.fits = M <= kSmallMP && K % 128 == 0 && K <= kGWarps * 16 * 32 && nbox <= kMaxBoxes &&
           chunks_per_cta <= 256 && gemv_smem_bytes(nbox, p.mt) <= kSmemLimit;
  return p;
}

cudaError_t launch_few_quant(const GemvArgs& a, const GemvPlan& p, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.quant_ctas);
  cfg.blockDim = dim3(kQThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.quant_ctas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return p.mt == 8 ? cudaLaunchKernelEx(&cfg, few_quant_kernel<8>, a)
                   : cudaLaunchKernelEx(&cfg, few_quant_kernel<kSmallMP>, a);
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
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = gemv_smem_bytes(p.stages, p.mt);
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
