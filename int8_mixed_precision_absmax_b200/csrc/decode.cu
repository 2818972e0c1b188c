// decode.cu -- the LLM.int8() layer for up to 8 tokens in one launch (the decode regime).
//
// With M <= 8 the layer reads every byte of Wq once and does at most 8 multiply-adds per
// byte, so its time is the weight stream and the latency of the few steps that depend on X.
// One launch does the whole layer, built so that back-to-back layers keep HBM busy and the
// X-dependent chain stays short:
//
//   * A thread-block cluster of 8 CTAs owns a group of G output channels (G = 128, or 64
//     for K > 4096) and splits K eight ways: CTA r owns the r-th eighth of the 128-byte
//     k-blocks.  Its Wq tile (G rows x K/8 bytes, 64 KB) is copied by TMA into shared memory,
//     one box per 16-channel MMA tile, before the CTA waits for the previous launch on the
//     stream; the CTA then lets the next launch start.  A CTA needs about 70 KB of shared
//     memory, so CTAs of the next layer sit beside this layer's and stream their weights
//     while this layer computes.
//   * CTA r reads only its slice of X.  It finds the outlier columns of the slice,
//     max_i |x| > threshold ([P2] "8位量化实战：离群值处理与显存优化避坑指南" section 2.3)
//     -- a column lies in one slice, so this needs no exchange -- and the row maxima over its
//     regular columns.  The eight CTAs exchange those maxima through distributed shared
//     memory, giving sx = max / 127 per row, and each writes q = rne(x / sx) clamped to
//     [-127, 127], 0 in outlier columns ([P5] "PyTorch 2.9 支持 LLM.int8()" item 2), for its
//     own slice into its own shared memory.
//   * Each warp takes one 16-channel tile (and for K > 4096 half of the slice's k-steps) and
//     forms acc[n, i] = sum_k Wq[n,k] q[i,k] exactly with the int8 warp-level MMA m16n8k32
//     (16 channels x 8 tokens; a tcgen05 MMA takes the same time at N = 8 tokens as at
//     N = 256, so at this shape it would idle).  In a k-step holding an outlier column it
//     also runs the fp16 MMA m16n8k16 on W_hat = fp16(Wq * w_scale) and the fp16 activations
//     of the outlier columns (zero elsewhere): the fp16 term of the decomposition, with fp32
//     accumulation ([P5] "如何在 PyTorch 2.9 中启用 LLM.int8 推理": no fp16 weights kept).
//   * The partial sums of the eight slices meet through distributed shared memory: CTA r
//     sums channels [r G/8, (r+1) G/8) over the cluster in a fixed order and writes
//     Y = fp16(acc * sx * w_scale + P + bias).
//
// Each thread's fragments cover 8 consecutive bytes of K per 32-wide k-step (the MMA's k
// positions are permuted the same way in both operands, which leaves the dot product as it
// is), so a fragment is one 8-byte shared-memory load.
//
// The weights and scales are read before the wait on the previous launch: they must not be
// written by the launch just before this one on the stream while it can still be running.
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kDThreads = 256;
constexpr int kDWarps = kDThreads / 32;
constexpr int kDTok = 8;               // tokens (MMA N)
constexpr int kDSplit = 8;             // CTAs per cluster = slices of K
constexpr int kDMaxKb = 64;            // K <= 8192
constexpr int kDMaxItems = 2;          // (chunk, token pair) items of the slice per thread
constexpr size_t kDSmemBudget = 74 * 1024;  // three CTAs per SM

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Split cluster barrier (per thread): every thread of the cluster arrives once per phase and
// waits before arriving again.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
// Arrive without ordering this thread's earlier memory operations: for the exit barrier, whose
// only job is to keep this CTA's shared memory alive while its peers still read it (each
// thread has used the values of its remote loads before it arrives), and for the threads of a
// CTA whose shared-memory writes thread 0 releases for all of them after a __syncthreads
// (release is cumulative).
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
// After a __syncthreads: warp 0 releases the CTA's shared-memory writes for all threads, the
// other warps arrive relaxed.  Every warp takes one branch as a whole: a warp never splits
// its arrival across two barrier instructions.
__device__ __forceinline__ void cluster_arrive_cta() {
  if (threadIdx.x < 32) cluster_arrive();
  else cluster_arrive_relaxed();
}
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Remote shared-memory stores and loads, ordered against the other side by a cluster barrier
// (volatile: they must not move across it).  Callers issue a batch of loads before using any
// result.
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Ask L2 to fetch `bytes` (a multiple of 16) at a 16-byte aligned global address.  L2 is where
// global memory is kept coherent, so this is safe even for data the previous launch may still
// be writing: its stores land in the same L2 lines; the data is read only after the wait.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

__device__ __forceinline__ float h2f(uint32_t word, int hi) {
  return __half2float(
      __ushort_as_half(static_cast<unsigned short>(hi ? (word >> 16) : (word & 0xFFFFu))));
}

// 8 codes of one row chunk, packed little-endian, outlier columns (bits) set to 0.
// rne(x * r) with r = 1/sx rounded to nearest equals rne(fl(x / sx)) unless x * r lies within
// 2^-15 of a half-integer (the exact x * r is within 2^-17 of x / sx for |x / sx| <= 128, the
// rounded quotient within 2^-18); there the quotient itself (__fdiv_rn) is rounded.
// tb = fl(x * r + 1.5 * 2^23) = 1.5 * 2^23 + rne(x * r) exactly, and as 1.5 * 2^23 has a zero
// low byte, the low byte of tb's bits is the two's-complement code.  d = x * r - rne(x * r)
// (one more FMA, rounding error <= 2^-25) has |d| <= 1/2, so "near a half-integer" is
// |d| > 1/2 - 2^-15.  A regular column has |x| <= the row maximum, so |x / sx| <=
// 127 (1 + 2^-22) and the code needs no clamp; outlier columns are masked out after the fact.
__device__ __forceinline__ uint32_t keep_mask(uint32_t bits4) {  // bit e set -> byte e = 0
  return ~(((bits4 * 0x204081u) & 0x01010101u) * 0xFFu);
}
__device__ __forceinline__ uint2 quantize8(const uint4& v, float sc, float rcp, uint32_t bits) {
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
        qb[e] = static_cast<uint32_t>(__float2int_rn(__fdiv_rn(x[e], sc)));
    }
  }
  const uint32_t lo = __byte_perm(__byte_perm(qb[0], qb[1], 0x0040), __byte_perm(qb[2], qb[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(qb[4], qb[5], 0x0040), __byte_perm(qb[6], qb[7], 0x0040), 0x5410);
  return make_uint2(lo & keep_mask(bits & 0xFu), hi & keep_mask(bits >> 4));
}

// D(16 x 8, int32) += A(16 x 32, int8, row-major) * B(32 x 8, int8, column-major)
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(16 x 8, fp32) += A(16 x 16, fp16, row-major) * B(16 x 8, fp16, column-major)
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp16(float(code) * scale) for bytes (2h, 2h+1) of an int8 word, packed as a half2 word
__device__ __forceinline__ uint32_t what2(uint32_t word, int h, float scale) {
  const float lo = static_cast<float>(static_cast<int8_t>((word >> (16 * h)) & 0xFFu));
  const float hi = static_cast<float>(static_cast<int8_t>((word >> (16 * h + 8)) & 0xFFu));
  const __half2 v = __halves2half2(__float2half_rn(__fmul_rn(lo, scale)),
                                   __float2half_rn(__fmul_rn(hi, scale)));
  return *reinterpret_cast<const uint32_t*>(&v);
}

// keep the halves of `word` (columns 2h, 2h+1 of a chunk) whose outlier bits are set
__device__ __forceinline__ uint32_t mask2(uint32_t word, uint32_t bits, int h) {
  const uint32_t lo = ((bits >> (2 * h)) & 1u) ? 0x0000FFFFu : 0u;
  const uint32_t hi = ((bits >> (2 * h + 1)) & 1u) ? 0xFFFF0000u : 0u;
  return word & (lo | hi);
}

struct DecodeShared {
  uint64_t full[kDWarps];      // one weight box per 16-channel tile
  float part[kDWarps][kDTok];   // row maxima of this CTA's slice, per warp
  float all_max[kDSplit][kDTok];  // row maxima of every slice (written by the slice's CTA)
  float sx[kDTok];
  float rcp[kDTok];
  int zero_row[kDTok];
  uint8_t flags[kDMaxKb / kDSplit * 16];  // outlier bits of the slice's 8-column chunks
  int abort;
};

// [Wq tiles: tiles x 16 rows x nqmax k-blocks x 128 B | int8 codes: 8 rows x (nqmax x 128
//  + 32) B]
size_t decode_smem_bytes(int tiles, int nqmax) {
  return 1024 + static_cast<size_t>(tiles) * 16 * 128 * nqmax +
         static_cast<size_t>(kDTok) * (128 * nqmax + 32);
}

// P = pairs of 16-channel tiles per CTA; the 8 warps are P pairs x (8 / P) parts of the
// slice's k-blocks.
template <int P>
__global__ void __launch_bounds__(kDThreads, 3)
    decode_kernel(const __grid_constant__ CUtensorMap map_wq, const DecodeArgs a) {
  constexpr int kParts = kDWarps / P;   // k-parts of the slice
  constexpr int kTiles = 2 * P;         // 16-channel tiles per CTA (and per cluster)
  constexpr int kG = 16 * kTiles;       // channels per cluster
  constexpr int kRed = kG / kDSplit;    // channels each CTA finishes
  extern __shared__ uint8_t decode_smem_raw[];
  __shared__ DecodeShared sh;
  uint8_t* wt = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(decode_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int nqmax = a.nqmax;
  const int tile_bytes = 16 * 128 * nqmax;
  uint8_t* xq_s = wt + kTiles * tile_bytes;  // [token][xq_ld] int8
  const int xq_ld = nqmax * 128 + 32;        // +32: the 8 token rows start in different banks
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int r = static_cast<int>(cluster_rank());
  const int n0 = (blockIdx.x / kDSplit) * kG;
  const int M = a.M, K = a.K, N = a.N;
  const int KB = K / 128;
  const int lo = r * KB / kDSplit, nq = (r + 1) * KB / kDSplit - lo;  // this CTA's k-blocks
  volatile int* abort = &sh.abort;

  if (tid == 0) {
    for (int t = 0; t < kTiles; ++t) mbar_init(&sh.full[t], 1);
    sh.abort = 0;
    fence_mbarrier_init();
    prefetch_tmap(&map_wq);
  }
  __syncthreads();
  if (tid == 0 && nq > 0) {  // the weight stream starts before the previous launch ends
    for (int t = 0; t < kTiles; ++t) {
      mbar_arrive_expect_tx(&sh.full[t], static_cast<uint32_t>(tile_bytes));
      tma_load_3d(&map_wq, wt + static_cast<size_t>(t) * tile_bytes, &sh.full[t], 0,
                  n0 + 16 * t, lo);
    }
  }
  const int g = lane >> 2, tig = lane & 3;
  const int pair = warp / kParts, part = warp % kParts;  // tiles 2 pair, 2 pair + 1
  float swr[2][2];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = n0 + 32 * pair + 16 * m + 8 * h + g;
      swr[m][h] = n < N ? a.w_scale[n] : 0.0f;
    }
  if (tid < M && nq > 0) prefetch_l2(a.X + static_cast<size_t>(tid) * K + lo * 128, nq * 256);
  grid_launch_dependents();
  grid_dependency_wait();  // X (the previous layer's output) is complete from here on

  // ---- this CTA's slice of X.  Item (chunk c of 8 columns, token pair p): the 4 lanes of
  // a chunk hold its 8 tokens.  The raw values stay in registers for the quantization.
  const int p = lane & 3;
  const int col0 = lo * 128;
  float rm0 = 0.0f, rm1 = 0.0f;  // row maxima of tokens 2p, 2p+1 over regular columns
  uint4 xv[kDMaxItems][2];
  uint32_t xbits[kDMaxItems];
#pragma unroll
  for (int it = 0; it < kDMaxItems; ++it) {
    const int item = tid + it * kDThreads;
    xbits[it] = 0u;
    xv[it][0] = xv[it][1] = make_uint4(0u, 0u, 0u, 0u);
    if (item < nq * 64) {  // warp-uniform: nq * 64 is a multiple of 64
      const int c = item >> 2;
      const int col = col0 + c * 8;
      if (2 * p < M)
        xv[it][0] = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(2 * p) * K + col));
      if (2 * p + 1 < M)
        xv[it][1] = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(2 * p + 1) * K + col));
      const uint32_t w0[4] = {xv[it][0].x, xv[it][0].y, xv[it][0].z, xv[it][0].w};
      const uint32_t w1[4] = {xv[it][1].x, xv[it][1].y, xv[it][1].z, xv[it][1].w};
      uint32_t bits = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2 m = __hmax2(__habs2(*reinterpret_cast<const __half2*>(&w0[e])),
                            __habs2(*reinterpret_cast<const __half2*>(&w1[e])));
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          const uint32_t other = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t*>(&m), o);
          m = __hmax2(m, *reinterpret_cast<const __half2*>(&other));
        }
        if (__low2float(m) > a.threshold) bits |= 1u << (2 * e);
        if (__high2float(m) > a.threshold) bits |= 1u << (2 * e + 1);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if ((bits >> e) & 1u) continue;
        rm0 = fmaxf(rm0, fabsf(h2f(w0[e / 2], e & 1)));
        rm1 = fmaxf(rm1, fabsf(h2f(w1[e / 2], e & 1)));
      }
      xbits[it] = bits;
      if (p == 0) sh.flags[c] = static_cast<uint8_t>(bits);
    }
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    rm0 = fmaxf(rm0, __shfl_xor_sync(0xffffffffu, rm0, o));
    rm1 = fmaxf(rm1, __shfl_xor_sync(0xffffffffu, rm1, o));
  }
  if (lane < 4) {
    sh.part[warp][2 * p] = rm0;
    sh.part[warp][2 * p + 1] = rm1;
  }
  __syncthreads();
  if (warp == 0) {
    // this slice's row maxima into every CTA of the cluster (lane: token lane % 8, CTAs
    // lane / 8 and lane / 8 + 4); warp 0's release below covers its own remote stores
    const int i = lane % kDTok;
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) m = fmaxf(m, sh.part[w][i]);
    const uint32_t local = smem_addr(&sh.all_max[r][i]);
#pragma unroll
    for (int h = 0; h < 2; ++h) st_cluster_f32(map_rank(local, lane / kDTok + 4 * h), m);
  }
  cluster_arrive_cta();

  // this warp's k-blocks and the k-steps among them holding an outlier column (bit
  // 4 (kb - kb_begin) + j); the fp16 activations of the first two such steps are fetched now,
  // while the cluster exchanges its row maxima
  const int kb_begin = part * nq / kParts, kb_end = (part + 1) * nq / kParts;
  const int nsteps = 4 * (kb_end - kb_begin);
  const uint32_t ow = lane < nsteps
      ? *reinterpret_cast<const uint32_t*>(&sh.flags[(4 * kb_begin + lane) * 4]) : 0u;
  const uint32_t outlier_steps = __ballot_sync(0xffffffffu, ow != 0u);
  const __half* xg = a.X + static_cast<size_t>(g) * K + col0 + 8 * tig;
  uint4 xo_pre[2];
  {
    uint32_t rest = outlier_steps;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      xo_pre[n] = make_uint4(0u, 0u, 0u, 0u);
      if (rest != 0u) {
        const int st = __ffs(rest) - 1;
        rest &= rest - 1u;
        if (g < M)
          xo_pre[n] = __ldg(reinterpret_cast<const uint4*>(xg + (kb_begin + st / 4) * 128 + 32 * (st % 4)));
      }
    }
  }
  cluster_wait();  // every slice's row maxima are in its shared memory

  if (tid < kDTok) {
    float m = 0.0f;
#pragma unroll
    for (int s = 0; s < kDSplit; ++s) m = fmaxf(m, sh.all_max[s][tid]);
    const float sc = __fdiv_rn(m, 127.0f);
    sh.sx[tid] = tid < M ? sc : 0.0f;
    sh.rcp[tid] = (tid < M && m > 0.0f) ? __frcp_rn(sc) : 0.0f;
    sh.zero_row[tid] = (tid >= M) || m == 0.0f;
  }
  __syncthreads();
  // ---- int8 codes of the slice: xq_s[token][column of the slice]
#pragma unroll
  for (int it = 0; it < kDMaxItems; ++it) {
    const int item = tid + it * kDThreads;
    if (item < nq * 64) {
      const int c = item >> 2;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = 2 * p + h;
        const uint2 code = sh.zero_row[i] ? make_uint2(0u, 0u)
                                          : quantize8(xv[it][h], sh.sx[i], sh.rcp[i], xbits[it]);
        *reinterpret_cast<uint2*>(xq_s + i * xq_ld + c * 8) = code;
      }
    }
  }
  __syncthreads();

  // ---- this warp: tiles 2 pair + m (m = 0, 1) over k-blocks [kb_begin, kb_end)
  int d[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
  float pf[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
  bool ok = true;
  if (kb_begin < kb_end) {
    bool landed = true;
    if (lane == 0)
      landed = mbar_wait_bounded(&sh.full[2 * pair], 0, abort) &&
               mbar_wait_bounded(&sh.full[2 * pair + 1], 0, abort);
    ok = __shfl_sync(0xffffffffu, landed ? 1 : 0, 0) != 0;
    mbar_try_wait(&sh.full[2 * pair], 0);  // each lane observes the completed phases
    mbar_try_wait(&sh.full[2 * pair + 1], 0);
  }
  if (ok && kb_begin < kb_end) {
    // rows g and g + 8 of the swizzled 16 x 128 tiles: one address per k-step of a k-block
    const uint8_t* wrow[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        wrow[m][j] = wt + (2 * pair + m) * tile_bytes + g * 128 +
                     (((2 * j + (tig >> 1)) ^ g) << 4) + (tig & 1) * 8 + kb_begin * (16 * 128);
    const uint8_t* xrow = xq_s + g * xq_ld + 8 * tig + kb_begin * 128;
    int n_out = 0;
    for (int kb = kb_begin; kb < kb_end; ++kb) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint2 xb = *reinterpret_cast<const uint2*>(xrow + 32 * j);
        uint2 w[2][2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          w[m][0] = *reinterpret_cast<const uint2*>(wrow[m][j]);
          w[m][1] = *reinterpret_cast<const uint2*>(wrow[m][j] + 1024);
          mma_s8_16832(d[m], w[m][0].x, w[m][1].x, w[m][0].y, w[m][1].y, xb.x, xb.y);
        }
        if ((outlier_steps >> ((kb - kb_begin) * 4 + j)) & 1u) {
          // fp16 term: this k-step's outlier columns only (the other activations are zero)
          const uint32_t fb = sh.flags[kb * 16 + 4 * j + tig];
          uint4 xr = n_out == 0 ? xo_pre[0] : xo_pre[1];
          if (n_out >= 2 && g < M) xr = __ldg(reinterpret_cast<const uint4*>(xg + kb * 128 + 32 * j));
          ++n_out;
          const uint32_t b0 = mask2(xr.x, fb, 0), b1 = mask2(xr.y, fb, 1);
          const uint32_t b2 = mask2(xr.z, fb, 2), b3 = mask2(xr.w, fb, 3);
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            uint32_t ha[2][4];  // rows g, g + 8: fp16 weights of this step's 8 columns
            if (a.W16) {        // the layer's kept fp16 weights
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int n = n0 + 32 * pair + 16 * m + 8 * h + g;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (n < N)
                  v = __ldg(reinterpret_cast<const uint4*>(
                      a.W16 + static_cast<size_t>(n) * K + col0 + kb * 128 + 32 * j + 8 * tig));
                ha[h][0] = v.x; ha[h][1] = v.y; ha[h][2] = v.z; ha[h][3] = v.w;
              }
            } else {            // fp16(Wq * w_scale) from the resident int8 tile
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                ha[h][0] = what2(w[m][h].x, 0, swr[m][h]);
                ha[h][1] = what2(w[m][h].x, 1, swr[m][h]);
                ha[h][2] = what2(w[m][h].y, 0, swr[m][h]);
                ha[h][3] = what2(w[m][h].y, 1, swr[m][h]);
              }
            }
            mma_f16_16816(pf[m], ha[0][0], ha[1][0], ha[0][1], ha[1][1], b0, b1);
            mma_f16_16816(pf[m], ha[0][2], ha[1][2], ha[0][3], ha[1][3], b2, b3);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j) wrow[m][j] += 16 * 128;
      xrow += 128;
    }
  }
  if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
  // partial sums of this part of the slice into the weight area (every warp is done reading
  // it): stage_i / stage_p [warp][32 channels][8 tokens]
  __syncthreads();
  int32_t* stage_i = reinterpret_cast<int32_t*>(wt);
  float* stage_p = reinterpret_cast<float*>(wt + kDWarps * 32 * kDTok * sizeof(int32_t));
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int c0 = (warp * 32 + 16 * m + g) * kDTok + 2 * tig, c1 = c0 + 8 * kDTok;
    stage_i[c0] = d[m][0];
    stage_i[c0 + 1] = d[m][1];
    stage_i[c1] = d[m][2];
    stage_i[c1 + 1] = d[m][3];
    stage_p[c0] = pf[m][0];
    stage_p[c0 + 1] = pf[m][1];
    stage_p[c1] = pf[m][2];
    stage_p[c1 + 1] = pf[m][3];
  }
  __syncthreads();
  // sum over the k-parts of each tile pair, in place into the part-0 slots: stage[pair * kParts]
  for (int e = tid; e < P * 32 * kDTok; e += kDThreads) {
    const int pr = e / (32 * kDTok), off = e % (32 * kDTok);
    int32_t si = stage_i[(pr * kParts) * 32 * kDTok + off];
    float sp = stage_p[(pr * kParts) * 32 * kDTok + off];
#pragma unroll
    for (int h = 1; h < kParts; ++h) {
      si += stage_i[(pr * kParts + h) * 32 * kDTok + off];
      sp += stage_p[(pr * kParts + h) * 32 * kDTok + off];
    }
    stage_i[(pr * kParts) * 32 * kDTok + off] = si;
    stage_p[(pr * kParts) * 32 * kDTok + off] = sp;
  }
  __syncthreads();
  cluster_arrive_cta();
  cluster_wait();  // every slice's partial sums are in its shared memory

  // ---- CTA r finishes channels [r * kRed, (r + 1) * kRed) of the group.  Thread (channel,
  // token quad, kind) sums the int32 (kind 0) or fp32 (kind 1) partials of the 8 slices in a
  // fixed order; the two kinds meet through a shuffle.
  if (tid < 4 * kRed) {  // whole warps: 4 * kRed is 64 or 32
    const int kind = tid & 1, quad = (tid >> 1) & 1, cl = r * kRed + (tid >> 2);
    const int pr = cl / 32, cr = cl % 32;
    const uint8_t* stage = kind ? reinterpret_cast<const uint8_t*>(stage_p)
                                : reinterpret_cast<const uint8_t*>(stage_i);
    uint4 v[kDSplit];
    const uint32_t local = smem_addr(stage + ((((pr * kParts) * 32 + cr) * kDTok + 4 * quad) * 4));
#pragma unroll
    for (int q = 0; q < kDSplit; ++q) v[q] = ld_cluster_v4(map_rank(local, q));
    uint32_t sum[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int q = 0; q < kDSplit; ++q) {
      const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sum[e] = kind ? __float_as_uint(__uint_as_float(sum[e]) + __uint_as_float(w[e]))
                      : sum[e] + w[e];
    }
    uint32_t other[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) other[e] = __shfl_xor_sync(0xffffffffu, sum[e], 1);
    const int n = n0 + cl;
    if (kind == 0 && n < N) {
      const float swn = a.w_scale[n];
      const float bb = a.bias ? __half2float(a.bias[n]) : 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 4 * quad + e;
        if (i >= M) continue;
        const int acc = static_cast<int>(sum[e]);
        const float y = static_cast<float>(acc) * sh.sx[i] * swn + __uint_as_float(other[e]) + bb;
        a.Y[static_cast<size_t>(i) * N + n] = __float2half_rn(y);
        if (a.acc) a.acc[static_cast<size_t>(i) * N + n] = sh.abort ? 0 : acc;
      }
    }
  }
  cluster_arrive_relaxed();  // this CTA is done reading its peers' shared memory
  if (tid == 0 && nq > 0) {
    // every copy this CTA started has landed before it exits (normally long ago)
    int dummy = 0;
    for (int t = 0; t < kTiles; ++t) mbar_wait_bounded(&sh.full[t], 0, &dummy);
  }
  cluster_wait();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace

DecodePlan plan_decode(int M, int N, int K) {
  DecodePlan p = {};
  p.fits = false;
  if (M > kDTok || K % 128 != 0 || K / 128 > kDMaxKb || N <= 0) return p;
  const int KB = K / 128;
  p.cluster = kDSplit;
  p.nqmax = (KB + kDSplit - 1) / kDSplit;
  p.wpm = K <= 4096 ? 4 : 2;  // pairs of 16-channel tiles per CTA
  const int tiles = 2 * p.wpm;
  p.tile_rows = 16;
  p.smem = decode_smem_bytes(tiles, p.nqmax);
  const int groups = (N + 16 * tiles - 1) / (16 * tiles);
  p.ctas = groups * kDSplit;
  p.fits = p.smem + sizeof(DecodeShared) <= kDSmemBudget;
  return p;
}

cudaError_t launch_decode(const CUtensorMap& map_wq, const DecodeArgs& a, const DecodePlan& p,
                          cudaStream_t stream, bool pdl) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != configured_device) {
    e = cudaFuncSetAttribute(decode_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kDSmemBudget));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kDSmemBudget));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ctas);
  cfg.blockDim = dim3(kDThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return p.wpm == 4 ? cudaLaunchKernelEx(&cfg, decode_kernel<4>, map_wq, a)
                     : cudaLaunchKernelEx(&cfg, decode_kernel<2>, map_wq, a);
}

}  // namespace i8mm
