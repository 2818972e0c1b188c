// small.cu -- the LLM.int8() layer for a few tokens (M <= 16: the decode regime), in one
// kernel launch.
//
// With so few rows the layer is a weight-streaming problem: every byte of Wq must be read
// once at HBM speed and everything else hidden behind that stream.  Each output tile of
// 128 channels is computed by a thread-block cluster of S CTAs that split K (split-K).
// Each CTA of a cluster:
//   1. starts the TMA stream of its Wq slice [128 channels x K/S] into a ring of up to 8
//      stages (all of it, when the slice is that short);
//   2. reads its K-slice of X for all M rows and finds, per column, whether any |x|
//      exceeds the threshold (the outlier columns of [P2] "8位量化实战：离群值处理与显存
//      优化避坑指南" section 2.3 -- complete per slice, since every row is present) and,
//      per row, the largest |x| over the slice's regular columns;
//   3. after a cluster barrier, reads the other CTAs' row maxima from their shared memory
//      (distributed shared memory) to form the row scale sx = max / 127 over all of K
//      ([P5] "PyTorch 2.9 支持 LLM.int8()" item 2, taken over X_R), identical in every CTA;
//   4. quantizes its slice, q = rne(x / sx) clamped to [-127, 127] and 0 in outlier
//      columns, straight into the 128-byte-swizzled shared-memory layout of the MMA's B
//      operand, and one thread issues tcgen05.mma kind::i8 (M = 128 channels, N = 16
//      tokens, int32 accumulator in tensor memory);
//   5. meanwhile computes the fp16 outlier term of the outlier columns in its slice,
//      sum_j X[i,j] * fp16(Wq[n,j] * w_scale[n]) ([P5] "如何在 PyTorch 2.9 中启用 LLM.int8
//      推理": no fp16 weights are kept);
//   6. after a second cluster barrier, sums the S partial int32 accumulators and outlier
//      terms of its share of the channels from the cluster's shared memory, in rank order
//      (deterministic), and writes Y = fp16(acc * sx * w_scale + P + bias).
// No CTA waits on another except through the cluster's hardware barrier; the kernel keeps
// no state in global memory between calls.
//
// Quantization arithmetic: the codes of the IEEE quotient x / sx (codes.cuh).
#include "codes.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxStages = 8;
constexpr int kABytes = kSmallBN * kBKBytes;       // 16 KB of Wq per stage
constexpr int kBBytesPerKb = kSmallMP * kBKBytes;  // 2 KB of Xq per k-block
constexpr int kAccs = 4;               // independent accumulators, summed in the drain
constexpr uint32_t kTmemCols = 64;      // kAccs x 16 columns
constexpr uint32_t kIdesc = idesc_i8_s32(kSmallBN, kSmallMP);
constexpr int kStatThreads = 192;   // warps 2..7: statistics of the slice
constexpr int kQuantThreads = 128;  // warps 4..7: quantization and the accumulator drain

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Split cluster barrier (per thread, not warp-collective): every thread of every CTA of
// the cluster arrives once per phase and waits before arriving again.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
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

__device__ __forceinline__ float half_bits_to_float(uint32_t word, int hi) {
  return __half2float(
      __ushort_as_half(static_cast<unsigned short>(hi ? (word >> 16) : (word & 0xFFFFu))));
}

}  // namespace

struct SmallShared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t xq_ready;
  uint64_t tmem_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int epi_ok;
  int issued;
  float rowmax_local[kSmallMP];  // read by the other CTAs of the cluster
  float red[kStatThreads / 32][kSmallMP];
  float sx[kSmallMP];
  float rcp[kSmallMP];
  int zero_row[kSmallMP];
  uint8_t flags[kSmallMaxKbPerSplit * 16];  // outlier bits, 8 columns per byte
  int32_t acc[kSmallBN][kSmallMP];          // this CTA's partial sums, read cluster-wide
  float psum[kSmallBN][kSmallMP];           // this CTA's outlier term, read cluster-wide
  float wscale[kSmallBN];                   // the tile's w_scale and bias
  float bias[kSmallBN];
};

constexpr size_t kSmemLimit = 227 * 1024;

// [Wq ring | Xq tiles | X slice (M rows) | SmallShared]
size_t small_smem_bytes(int stages, int kb_per_split, int M) {
  return 1024 + static_cast<size_t>(stages) * kABytes +
         static_cast<size_t>(kb_per_split) * kBBytesPerKb +
         static_cast<size_t>(M) * kb_per_split * kBKBytes * sizeof(__half) + sizeof(SmallShared) + 16;
}

// The deepest ring (all of the slice when it fits) within the shared-memory limit.
int small_stages(int kb_per_split, int M) {
  int st = kb_per_split < kMaxStages ? kb_per_split : kMaxStages;
  while (st > 2 && small_smem_bytes(st, kb_per_split, M) > kSmemLimit) --st;
  return st;
}

__global__ void __launch_bounds__(kThreads, 1)
    small_fused_kernel(const __grid_constant__ CUtensorMap map_wq, const SmallArgs a) {
  extern __shared__ uint8_t small_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(small_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int S = a.splits;
  const int kb_total = (a.K + kBKBytes - 1) / kBKBytes;
  const int kb_max = (kb_total + S - 1) / S;  // the same in every CTA: a common smem layout
  const int kStages = a.stages;
  uint8_t* a_stage = base;                       // kStages x 16 KB
  uint8_t* xq_tiles = base + kStages * kABytes;  // kb_max x 2 KB
  const int split = static_cast<int>(cluster_rank());
  const int tile = blockIdx.x / S;
  const int n0 = tile * kSmallBN;
  const int kb_begin = static_cast<int>(static_cast<long long>(split) * kb_total / S);
  const int kb_end = static_cast<int>(static_cast<long long>(split + 1) * kb_total / S);
  const int nkb = kb_end - kb_begin;
  __half* x_slice = reinterpret_cast<__half*>(xq_tiles + kb_max * kBBytesPerKb);  // [M][kb_max*128]
  const int xs_ld = kb_max * kBKBytes;
  SmallShared& sh = *reinterpret_cast<SmallShared*>(x_slice + static_cast<size_t>(a.M) * xs_ld);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort = &sh.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    mbar_init(&sh.xq_ready, kQuantThreads);  // warps 4..7
    mbar_init(&sh.tmem_full, 1);
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    sh.issued = 0;
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
  // The inputs may be written by the previous launch on the stream: wait for it before
  // the first read (everything above overlapped its tail).
  grid_dependency_wait();

  if (warp == 0) {
    cluster_arrive();  // phase 1 (row maxima) needs nothing from this warp
    if (lane == 0) {
      // ---- TMA producer: the Wq slice, 128 channels x 128 bytes per stage
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < nkb; ++j) {
        const int s = j % kStages;
        if (j >= kStages &&
            !mbar_wait_bounded(&sh.empty[s], static_cast<uint32_t>((j / kStages) - 1) & 1u,
                               abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sh.full[s], kABytes);
        tma_load_2d(&map_wq, a_stage + s * kABytes, &sh.full[s], (kb_begin + j) * kBKBytes, n0);
        ++issued;
      }
      sh.issued = issued;  // the teardown drains these if any role gave up
      if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
    }
    cluster_wait();
    cluster_arrive();  // phase 2 (partial sums)
    cluster_wait();
  } else if (warp == 1) {
    cluster_arrive();
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
          for (int k = 0; k < 4; ++k)  // accumulator k: four independent chains
            mma_i8(tmem + static_cast<uint32_t>(k * kSmallMP), sw128_kmajor_desc(a0 + 32u * k),
                   sw128_kmajor_desc(b0 + 32u * k), kIdesc, j > 0 ? 1u : 0u);
          mma_commit(&sh.empty[s]);
        }
        if (ok) mma_commit(&sh.tmem_full);
      }
      mma_commit(&sh.drain);  // every MMA issued must finish before TMEM is freed
      int dummy = 0;
      mbar_wait_bounded(&sh.drain, 0, &dummy);
      if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
    }
    cluster_wait();
    cluster_arrive();
    cluster_wait();
  } else {
    // ---- warps 2..7: statistics of this K-slice of X.  Thread tq owns 8-column chunks
    // c = tq, tq + 192, ... for all rows; the slice is also staged in shared memory.
    const int tq = threadIdx.x - 64;  // 0..191
    const int col_begin = kb_begin * kBKBytes;
    const int chunks = nkb * (kBKBytes / 8);
    float rmax[kSmallMP];
#pragma unroll
    for (int i = 0; i < kSmallMP; ++i) rmax[i] = 0.0f;
    for (int c = tq; c < chunks; c += kStatThreads) {
      const int k = col_begin + c * 8;
      uint4 v[kSmallMP];
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) {
        v[i] = make_uint4(0u, 0u, 0u, 0u);
        if (i < a.M && k < a.K)
          v[i] = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * a.K + k));
      }
      __half2 cm[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) cm[e] = __float2half2_rn(0.0f);
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) {
        if (i < a.M) *reinterpret_cast<uint4*>(x_slice + static_cast<size_t>(i) * xs_ld + c * 8) = v[i];
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
      sh.flags[c] = static_cast<uint8_t>(bits);
      if (a.trace.flags && tile == 0 && kb_begin * 16 + c < 4 * ((a.K + 31) / 32))
        a.trace.flags[kb_begin * 16 + c] = static_cast<uint8_t>(bits);
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (!((bits >> e) & 1u))
            rmax[i] = fmaxf(rmax[i], fabsf(half_bits_to_float(w[e / 2], e & 1)));
      }
    }
    // row maxima of this slice: warp then block reduction
#pragma unroll
    for (int i = 0; i < kSmallMP; ++i) {
      float m = rmax[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      rmax[i] = m;
    }
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) sh.red[warp - 2][i] = rmax[i];
    }
    if (tq < kSmallBN) {
      const int gn = n0 + tq;
      sh.wscale[tq] = gn < a.N ? a.w_scale[gn] : 0.0f;
      sh.bias[tq] = (a.bias && gn < a.N) ? __half2float(a.bias[gn]) : 0.0f;
    }
    named_barrier(1, kStatThreads);  // flags, x_slice, red, wscale and bias are complete
    if (tq < kSmallMP) {
      float m = 0.0f;
#pragma unroll
      for (int w = 0; w < kStatThreads / 32; ++w) m = fmaxf(m, sh.red[w][tq]);
      sh.rowmax_local[tq] = m;
    }
    cluster_arrive();  // phase 1: every CTA's rowmax_local is written

    if (warp < 4) {
      // ---- warps 2..3: the fp16 outlier term of the outlier columns in this slice,
      // P[n][i] = sum_j X[i,j] * fp16(Wq[n0+n, j] * w_scale[n0+n]), channels tq and tq + 64.
      // It needs no row scale, so it runs while the cluster agrees on the scales.
      float P0[kSmallMP], P1[kSmallMP];
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) P0[i] = P1[i] = 0.0f;
      const int g0 = n0 + tq, g1 = n0 + tq + 64;
      const float s0 = sh.wscale[tq], s1 = sh.wscale[tq + 64];
      const int8_t* w0row = a.Wq + static_cast<size_t>(g0 < a.N ? g0 : 0) * a.K;
      const int8_t* w1row = a.Wq + static_cast<size_t>(g1 < a.N ? g1 : 0) * a.K;
      // With the whole slice resident in the ring (no stage is reused), the weights of an
      // outlier column are read from the landed TMA tile instead of from HBM.
      const bool resident = nkb <= kStages;
      for (int c = 0; c < chunks; ++c) {
        uint32_t bits = sh.flags[c];
        while (bits) {
          const int jl = c * 8 + __ffs(bits) - 1;  // column within the slice
          const int j = col_begin + jl;
          bits &= bits - 1u;
          int8_t q0, q1;
          if (resident) {
            const int kbl = jl / kBKBytes, kk = jl % kBKBytes;
            mbar_wait_bounded(&sh.full[kbl], 0, abort);
            const uint8_t* tile = a_stage + kbl * kABytes;
            q0 = static_cast<int8_t>(tile[(tq / 8) * 1024 + (tq % 8) * 128 +
                                          (((kk / 16) ^ (tq % 8)) * 16) + kk % 16]);
            const int t1 = tq + 64;
            q1 = static_cast<int8_t>(tile[(t1 / 8) * 1024 + (t1 % 8) * 128 +
                                          (((kk / 16) ^ (t1 % 8)) * 16) + kk % 16]);
          } else {
            q0 = w0row[j];
            q1 = w1row[j];
          }
          float w0 = __half2float(__float2half_rn(static_cast<float>(q0) * s0));
          float w1 = __half2float(__float2half_rn(static_cast<float>(q1) * s1));
          if (a.W16) {  // the layer's kept fp16 weights of the outlier column
            w0 = g0 < a.N ? __half2float(a.W16[static_cast<size_t>(g0) * a.K + j]) : 0.0f;
            w1 = g1 < a.N ? __half2float(a.W16[static_cast<size_t>(g1) * a.K + j]) : 0.0f;
          }
          if (a.trace.what) {  // the weights this term multiplies, as fp16
            if (g0 < a.N) a.trace.what[static_cast<size_t>(g0) * a.K + j] = __float2half_rn(w0);
            if (g1 < a.N) a.trace.what[static_cast<size_t>(g1) * a.K + j] = __float2half_rn(w1);
          }
          const __half* xc = x_slice + (j - col_begin);
#pragma unroll
          for (int i = 0; i < kSmallMP; ++i)
            if (i < a.M) {
              const float xv = __half2float(xc[static_cast<size_t>(i) * xs_ld]);
              P0[i] += w0 * xv;
              P1[i] += w1 * xv;
            }
        }
      }
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) {
        sh.psum[tq][i] = P0[i];
        sh.psum[tq + 64][i] = P1[i];
      }
      cluster_wait();
    } else {
      // ---- warps 4..7: the row scales, then quantize the slice into the B operand
      const int tz = threadIdx.x - 128;  // 0..127
      cluster_wait();
      if (tz < kSmallMP) {
        const uint32_t local = smem_addr(&sh.rowmax_local[tz]);
        float peer[kSmallMaxSplits];
#pragma unroll
        for (int r = 0; r < kSmallMaxSplits; ++r)  // all remote loads in flight at once
          peer[r] = r < S ? ld_cluster_f32(map_rank(local, r)) : 0.0f;
        float m = 0.0f;
#pragma unroll
        for (int r = 0; r < kSmallMaxSplits; ++r) m = fmaxf(m, peer[r]);
        if (a.per_tensor)  // one scale for all rows: the largest row absmax (rows past M hold 0)
#pragma unroll
          for (int o = 1; o < kSmallMP; o <<= 1)
            m = fmaxf(m, __shfl_xor_sync((1u << kSmallMP) - 1u, m, o));
        const float sc = __fdiv_rn(m, 127.0f);
        sh.sx[tz] = (tz < a.M) ? sc : 0.0f;
        sh.rcp[tz] = (tz < a.M && m > 0.0f) ? __frcp_rn(sc) : 0.0f;
        sh.zero_row[tz] = (tz >= a.M) || m == 0.0f;
        if (a.trace.sx && tile == 0 && split == 0 && tz < a.M) a.trace.sx[tz] = sc;
      }
      named_barrier(2, kQuantThreads);
      // thread tz quantizes chunk c (8 columns) for all 16 rows, independently per row;
      // codes for row i, k-block kbl, byte kk go to
      //   kbl*2048 + (i/8)*1024 + (i%8)*128 + ((kk/16) ^ (i%8))*16 + kk%16
      for (int c = tz; c < chunks; c += kQuantThreads) {
        const uint32_t bits = sh.flags[c];
        const int kbl = c / 16, kk = (c % 16) * 8;
        uint8_t* tile = xq_tiles + kbl * kBBytesPerKb + (kk % 16);
#pragma unroll
        for (int i = 0; i < kSmallMP; ++i) {
          uint2 q = make_uint2(0u, 0u);
          if (!sh.zero_row[i]) {
            const uint4 v =
                *reinterpret_cast<const uint4*>(x_slice + static_cast<size_t>(i) * xs_ld + c * 8);
            const uint2 c8 = codes8(v, sh.sx[i], sh.rcp[i]);
            const uint2 keep = keep_bytes(bits);
            q = make_uint2(c8.x & keep.x, c8.y & keep.y);
          }
          *reinterpret_cast<uint2*>(tile + (i / 8) * 1024 + (i % 8) * 128 +
                                    (((kk / 16) ^ (i % 8)) * 16)) = q;
          const int kg = col_begin + c * 8;  // the chunk's first column in X
          if (a.trace.xq && blockIdx.x < static_cast<unsigned>(S) && i < a.M && kg < a.K)
            *reinterpret_cast<uint2*>(a.trace.xq + static_cast<size_t>(i) * a.K + kg) = q;
        }
      }
      fence_async_shared();
      mbar_arrive(&sh.xq_ready);

      // ---- drain the accumulator: TMEM lane quadrant q <-> channels 32q .. 32q+31
      const int quad = warp & 3;
      const int n = quad * 32 + lane;
      mbar_wait_bounded(&sh.tmem_full, 0, abort);
      // one decision for the 128 threads
      named_barrier(2, kQuantThreads);
      if (threadIdx.x == 128) sh.epi_ok = (*abort == 0);
      named_barrier(2, kQuantThreads);
      tc_fence_after();
      int32_t accs[kSmallMP];
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) accs[i] = 0;
      __syncwarp();
#pragma unroll
      for (int k = 0; k < kAccs; ++k) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                               static_cast<uint32_t>(k * kSmallMP), r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < kSmallMP; ++i) accs[i] += static_cast<int32_t>(r[i]);
      }
      const bool ok = sh.epi_ok != 0;
#pragma unroll
      for (int i = 0; i < kSmallMP; ++i) sh.acc[n][i] = ok ? accs[i] : 0;
      if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
    }
    cluster_arrive();  // phase 2: every CTA's partial sums are in its shared memory
    cluster_wait();
    // ---- sum the S partials of this CTA's share of the output, in rank order
    const int outs = kSmallBN * a.M;
    const int per = (outs + S - 1) / S;
    const int o_begin = split * per, o_end = min(outs, o_begin + per);
    for (int o = o_begin + tq; o < o_end; o += kStatThreads) {
      const int n = o / a.M, i = o % a.M, gn = n0 + n;
      if (gn >= a.N) continue;
      const uint32_t acc_l = smem_addr(&sh.acc[n][i]);
      const uint32_t p_l = smem_addr(&sh.psum[n][i]);
      int32_t pa[kSmallMaxSplits];
      float pp[kSmallMaxSplits];
#pragma unroll
      for (int r = 0; r < kSmallMaxSplits; ++r) {  // all remote loads in flight at once
        pa[r] = r < S ? ld_cluster_s32(map_rank(acc_l, r)) : 0;
        pp[r] = r < S ? ld_cluster_f32(map_rank(p_l, r)) : 0.0f;
      }
      int32_t acc = 0;
      float P = 0.0f;
#pragma unroll
      for (int r = 0; r < kSmallMaxSplits; ++r) {  // rank order: the same bits every call
        acc += pa[r];
        P += pp[r];
      }
      const float y = static_cast<float>(acc) * sh.sx[i] * sh.wscale[n] + P + sh.bias[n];
      a.Y[static_cast<size_t>(i) * a.N + gn] = __float2half_rn(y);
      if (a.acc) a.acc[static_cast<size_t>(i) * a.N + gn] = acc;
    }
  }

  // no CTA may leave while the others can still read its shared memory
  cluster_arrive();
  cluster_wait();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && sh.abort) {
    // A wait gave up: the MMA thread may not have seen every stage land, so let the copies
    // still in flight finish before the shared memory is released.
    int dummy = 0;
    for (int d = sh.issued > kStages ? sh.issued - kStages : 0; d < sh.issued; ++d)
      mbar_wait_bounded(&sh.full[d % kStages], static_cast<uint32_t>(d / kStages) & 1u, &dummy);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

namespace {

int kb_per_split(int kb_total, int S) { return (kb_total + S - 1) / S; }

cudaError_t configure_small() {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev == configured_device) return cudaSuccess;
  e = cudaFuncSetAttribute(small_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemLimit));
  if (e == cudaSuccess) configured_device = dev;
  return e;
}

// Clusters of S CTAs that can be resident at once with this shared-memory footprint.
int max_active_clusters(int S, size_t smem) {
  struct Entry { int dev, S; size_t smem; int n; };
  static Entry cache[32];
  static int used = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  for (int i = 0; i < used; ++i)
    if (cache[i].dev == dev && cache[i].S == S && cache[i].smem == smem) return cache[i].n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, small_fused_kernel, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 1;
  }
  if (used < 32) cache[used++] = {dev, S, smem, n};
  return n;
}

}  // namespace

// Cluster size S (CTAs splitting K per 128-channel tile): the one that minimises
// (waves of resident clusters) x (k-blocks per CTA), preferring larger S on ties.
SmallPlan plan_small(int M, int N, int K) {
  SmallPlan p;
  p.tiles = (N + kSmallBN - 1) / kSmallBN;
  const int kb_total = (K + kBKBytes - 1) / kBKBytes;
  p.splits = 0;
  long long best = 0;
  if (configure_small() != cudaSuccess) cudaGetLastError();
  for (int S = kSmallMaxSplits; S >= 1; S /= 2) {
    if (S > kb_total) continue;
    const int kbps = kb_per_split(kb_total, S);
    if (kbps > kSmallMaxKbPerSplit) continue;
    const int act = max_active_clusters(S, small_smem_bytes(small_stages(kbps, M), kbps, M));
    const long long cost = static_cast<long long>((p.tiles + act - 1) / act) * kbps;
    if (p.splits == 0 || cost < best) {
      best = cost;
      p.splits = S;
    }
  }
  if (p.splits == 0) p.splits = 1;
  p.kb_per_split = kb_per_split(kb_total, p.splits);
  p.stages = small_stages(p.kb_per_split, M);
  return p;
}

bool small_path_fits(int M, int K) {
  if (M > kSmallMP) return false;
  const int kb_total = (K + kBKBytes - 1) / kBKBytes;
  const int S = kb_total < kSmallMaxSplits ? kb_total : kSmallMaxSplits;
  const int kbps = kb_per_split(kb_total, S);
  return kbps <= kSmallMaxKbPerSplit &&
         small_smem_bytes(small_stages(kbps, M), kbps, M) <= kSmemLimit;
}

cudaError_t launch_small(const CUtensorMap& map_wq, const SmallArgs& a, const SmallPlan& p,
                         cudaStream_t stream, bool pdl) {
  cudaError_t e = configure_small();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.tiles * p.splits);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = small_smem_bytes(p.stages, p.kb_per_split, a.M);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, small_fused_kernel, map_wq, a);
}

}  // namespace i8mm
