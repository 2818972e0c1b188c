// decode.cu -- the LLM.int8() layer for up to 8 tokens in one launch (the decode regime).
//
// With M <= 8 the layer reads every byte of Wq once and does at most 8 multiply-adds per
// byte, so its time is the weight stream plus the latency of the steps that depend on X.
// One launch does the whole layer, and every CTA works on its own, with no exchange between
// CTAs:
//
//   * A CTA owns 16 T output channels (T = 2 for K <= 4096, else 1) and all of K.  Its Wq
//     rows (16 T x K bytes, at most 128 KB) are copied by TMA into shared memory, one box
//     per 16-channel MMA tile, before the CTA waits for the previous launch on the stream;
//     the CTA then lets the next launch start.
//   * Each CTA reads the whole of X (8 x K fp16, 64 KB at K = 4096, from L2) and finds by
//     itself what the layer needs of it.  Thread t holds 8-column chunks of X for all 8
//     tokens in registers, so the column maxima need no exchange: a column is an outlier
//     when max_i |x| > threshold ([P2] "8位量化实战：离群值处理与显存优化避坑指南" section
//     2.3).  The row maxima over the regular columns meet in one block-wide reduction, giving
//     sx = max / 127 per row, and every thread writes q = rne(x / sx) in [-127, 127], 0 in
//     outlier columns ([P5] "PyTorch 2.9 支持 LLM.int8()" item 2), for its chunks into shared
//     memory.  Repeating this work in every CTA measured faster than sharing it across a
//     thread-block cluster (the remote stores and the cluster barrier cost more than the
//     quantization they save), and it runs while the weights are still arriving.
//   * Warp w takes the w-th sixteenth of the k-blocks for all T tiles and forms
//     acc[n, i] = sum_k Wq[n,k] q[i,k] exactly with the int8 warp-level MMA m16n8k32
//     (16 channels x 8 tokens; a CTA owns 32 channels, fewer than the 64 rows a tcgen05 MMA
//     needs).  Its k-steps holding an outlier column then run, one at a time, the fp16 MMA
//     m16n8k16 on the outlier weights and the fp16 activations of the outlier columns (zero
//     elsewhere, kept in shared memory since the statistics pass): the fp16 term of the
//     decomposition, with fp32 accumulation.  The outlier weights are W_hat =
//     fp16(Wq * w_scale) ([P5] "如何在 PyTorch 2.9 中启用 LLM.int8 推理",
//     has_fp16_weights=False), or the layer's own fp16 weights when it keeps them.
//   * The 16 warps' partial sums meet in shared memory; thread (token, channel) sums them in
//     a fixed order and writes Y = fp16(acc * sx * w_scale + P + bias).
//
// Each lane's fragments cover 8 consecutive bytes of K per 32-wide k-step, chosen so that the
// 16 lanes of a half-warp read 16 different bank pairs of the swizzled weight rows and of the
// codes (the MMA's k positions are permuted the same way in both operands, which leaves the
// dot product as it is); a fragment is one 8-byte shared-memory load.
//
// Wq is read before the wait on the previous launch (everything else after it): it must not
// be written by the launch just before this one on the stream while that can still be running.
#include "codes.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kDThreads = 512;
constexpr int kDWarps = kDThreads / 32;
constexpr int kDTok = 8;                // tokens (MMA N)
constexpr int kDMaxKb = 64;             // K <= 8192
constexpr int kDMaxTiles = 2;
constexpr int kDOutChunks = 64;         // 8-column chunks with an outlier kept in shared memory
constexpr size_t kDSmemMax = 227 * 1024;

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

// 8 codes of one row chunk, packed little-endian, then ANDed with `keep` (zero bytes in outlier
// columns): the IEEE quotient's codes (codes.cuh).
__device__ __forceinline__ uint2 keep_masks(uint32_t bits) { return keep_bytes(bits); }
__device__ __forceinline__ uint2 quantize8(const uint4& v, float sc, float rcp, uint2 keep) {
  const uint2 q = codes8(v, sc, rcp);
  return make_uint2(q.x & keep.x, q.y & keep.y);
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

// fp16(float(code) * scale) for bytes (2h, 2h+1) of an int8 word, packed as a half2 word.
// float(code) is read off the bits 0x4B0000vv with vv = code + 128 (the float 2^23 + vv, exact)
// less 2^23 + 128: a byte permute, a XOR and an add instead of integer-to-float conversions.
__device__ __forceinline__ float code_to_float(uint32_t word, uint32_t byte_sel) {
  uint32_t bits;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(bits) : "r"(word), "r"(0x4B000000u), "r"(byte_sel));
  return __uint_as_float(bits ^ 0x80u) - 8388736.0f;  // 2^23 + 128
}
__device__ __forceinline__ uint32_t what2(uint32_t word, int h, float scale) {
  // selector: byte 2h (or 2h + 1) of word, then bytes 1..3 of 0x4B000000
  const float lo = code_to_float(word, 0x7650u + 2u * h);
  const float hi = code_to_float(word, 0x7651u + 2u * h);
  const __half2 v = __floats2half2_rn(__fmul_rn(lo, scale), __fmul_rn(hi, scale));
  return *reinterpret_cast<const uint32_t*>(&v);
}

// keep the halves of `word` (columns 2h, 2h+1 of a chunk) whose outlier bits are set
__device__ __forceinline__ uint32_t mask2(uint32_t word, uint32_t bits, int h) {
  const uint32_t lo = ((bits >> (2 * h)) & 1u) ? 0x0000FFFFu : 0u;
  const uint32_t hi = ((bits >> (2 * h + 1)) & 1u) ? 0xFFFF0000u : 0u;
  return word & (lo | hi);
}

struct DecodeShared {
  uint64_t full[kDMaxTiles];    // one weight box per 16-channel tile
  uint4 part[kDWarps];          // per-warp row maxima: word e holds tokens 2e, 2e + 1 (fp16)
  float sx[kDTok];
  uint8_t flags[kDMaxKb * 16];  // outlier bits of each 8-column chunk of X
  uint8_t oslot[kDMaxKb * 16];  // chunk with an outlier -> its slot in xo (0xFF: not kept)
  uint4 xo[kDOutChunks][kDTok];  // fp16 X of the chunks with an outlier, per token
  int n_ochunks;
  int abort;
};

// partial sums of the 16 warps, [warp][token][stage_ld] per kind (int32, then fp32); the
// 4-word pad keeps the fragment stores free of bank conflicts
__host__ __device__ constexpr int stage_ld(int T) { return 16 * T + 4; }
__host__ __device__ constexpr int stage_bytes(int T) { return 2 * kDWarps * kDTok * stage_ld(T) * 4; }
// bytes of one tile: 16 rows x K/128 k-blocks x 128 B
__host__ __device__ inline int tile_bytes(int K) { return 16 * K; }
__host__ __device__ inline int weight_area(int T, int K) {
  return T * tile_bytes(K) > stage_bytes(T) ? T * tile_bytes(K) : stage_bytes(T);
}

// [Wq tiles: T x K/128 k-blocks x 16 rows x 128 B (or the staged sums) | codes: 8 x (K + 16) B]
size_t decode_smem_bytes(int T, int K) {
  return 1024 + static_cast<size_t>(weight_area(T, K)) + static_cast<size_t>(kDTok) * (K + 16);
}

// T 16-channel tiles per CTA; each thread holds up to kItems 8-column chunks of X.  kTrace:
// also write what the layer computed on the way (a.trace): CTA 0 the codes, the row scales
// and the outlier bits, every CTA its channels' fp16 weights at the outlier columns.
template <int T, int kItems, bool kTrace>
__global__ void __launch_bounds__(kDThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap map_wq, const DecodeArgs a) {
  constexpr int kC = 16 * T;  // channels per CTA
  constexpr int kLd = stage_ld(T);
  extern __shared__ uint8_t decode_smem_raw[];
  __shared__ DecodeShared sh;
  uint8_t* wt = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(decode_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int M = a.M, K = a.K, N = a.N;
  const int KB = K / 128;
  const int tb = tile_bytes(K);
  uint8_t* xq_s = wt + weight_area(T, K);  // [token][xq_ld] int8
  const int xq_ld = K + 16;                // +16: token rows g and g + 1 start 4 banks apart
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int g = lane >> 2, tig = lane & 3;
  const int n0 = blockIdx.x * kC;
  volatile int* abort = &sh.abort;

  if (tid < M) {  // CTA b asks L2 for the (b mod 8)-th eighth of each row of X, ahead of Wq
    const int seg = K / 8;
    prefetch_l2(a.X + static_cast<size_t>(tid) * K + (blockIdx.x % 8) * seg,
                static_cast<uint32_t>(seg * 2));
  }
  if (tid == 0) {
    for (int t = 0; t < T; ++t) mbar_init(&sh.full[t], 1);
    sh.abort = 0;
    sh.n_ochunks = 0;
    fence_mbarrier_init();
    prefetch_tmap(&map_wq);
  }
  __syncthreads();
  if (tid == 0) {  // the weight stream starts before the previous launch ends
    for (int t = 0; t < T; ++t) {
      mbar_arrive_expect_tx(&sh.full[t], static_cast<uint32_t>(tb));
      tma_load_3d(&map_wq, wt + static_cast<size_t>(t) * tb, &sh.full[t], 0, n0 + 16 * t, 0);
    }
  }
  grid_launch_dependents();
  grid_dependency_wait();  // X (the previous layer's output) is complete from here on
  float swr[T][2];  // scales of the fragment rows g, g + 8 of each tile
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = n0 + 16 * t + 8 * h + g;
      swr[t][h] = n < N ? a.w_scale[n] : 0.0f;
    }
  // the epilogue's (token, channel): thread tid < 8 kC
  const int ec = tid % kC, ei = tid / kC;
  const bool e_live = tid < kDTok * kC && ei < M && n0 + ec < N;
  const float e_sw = e_live ? a.w_scale[n0 + ec] : 0.0f;
  const float e_bias = (e_live && a.bias) ? __half2float(a.bias[n0 + ec]) : 0.0f;

  // ---- X: thread tid holds chunks c = tid + 512 u (8 columns x 8 tokens each) in registers
  const int chunks = K / 8;
  // fp16 x: |x| > t exactly when |x| > (t rounded down to fp16)
  const __half2 th2 = __half2half2(__float2half_rd(a.threshold));
  const __half2 zero2 = __float2half2_rn(0.0f);
  uint4 xv[kItems][kDTok];
  uint2 xkeep[kItems];
  __half2 rm[kDTok / 2];  // row maxima over regular columns, tokens (2e, 2e + 1)
#pragma unroll
  for (int e = 0; e < kDTok / 2; ++e) rm[e] = zero2;
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int c = tid + it * kDThreads;
    xkeep[it] = make_uint2(0u, 0u);
#pragma unroll
    for (int i = 0; i < kDTok; ++i) xv[it][i] = make_uint4(0u, 0u, 0u, 0u);
    if (c < chunks) {
#pragma unroll
      for (int i = 0; i < kDTok; ++i)
        if (i < M)
          xv[it][i] = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(i) * K + 8 * c));
      uint32_t keep[4];  // |x| of the regular columns: 0x7FFF per regular half, 0 per outlier
      uint32_t bits = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t cm = (&xv[it][0].x)[e] & 0x7FFF7FFFu;
#pragma unroll
        for (int i = 1; i < kDTok; ++i) {
          const uint32_t v = (&xv[it][i].x)[e] & 0x7FFF7FFFu;
          const __half2 m = __hmax2(*reinterpret_cast<const __half2*>(&cm),
                                    *reinterpret_cast<const __half2*>(&v));
          cm = *reinterpret_cast<const uint32_t*>(&m);
        }
        const uint32_t gt = __hgt2_mask(*reinterpret_cast<const __half2*>(&cm), th2);
        keep[e] = ~gt & 0x7FFF7FFFu;
        bits |= ((gt & 1u) | ((gt >> 15) & 2u)) << (2 * e);
      }
      xkeep[it] = keep_masks(bits);
      sh.flags[c] = static_cast<uint8_t>(bits);
      if (kTrace && blockIdx.x == 0 && a.trace.flags) a.trace.flags[c] = static_cast<uint8_t>(bits);
      if (bits != 0u) {  // keep the chunk's fp16 values for the outlier term
        const int slot = atomicAdd(&sh.n_ochunks, 1);
        sh.oslot[c] = static_cast<uint8_t>(slot < kDOutChunks ? slot : 0xFF);
        if (slot < kDOutChunks)
#pragma unroll
          for (int i = 0; i < kDTok; ++i) sh.xo[slot][i] = xv[it][i];
      }
#pragma unroll
      for (int i = 0; i < kDTok; i += 2) {
        uint32_t m0 = (&xv[it][i].x)[0] & keep[0], m1 = (&xv[it][i + 1].x)[0] & keep[0];
#pragma unroll
        for (int e = 1; e < 4; ++e) {
          const uint32_t v0 = (&xv[it][i].x)[e] & keep[e], v1 = (&xv[it][i + 1].x)[e] & keep[e];
          const __half2 h0 = __hmax2(*reinterpret_cast<const __half2*>(&m0),
                                     *reinterpret_cast<const __half2*>(&v0));
          const __half2 h1 = __hmax2(*reinterpret_cast<const __half2*>(&m1),
                                     *reinterpret_cast<const __half2*>(&v1));
          m0 = *reinterpret_cast<const uint32_t*>(&h0);
          m1 = *reinterpret_cast<const uint32_t*>(&h1);
        }
        const __half2 h0 = *reinterpret_cast<const __half2*>(&m0);
        const __half2 h1 = *reinterpret_cast<const __half2*>(&m1);
        rm[i / 2] = __hmax2(rm[i / 2], __halves2half2(__hmax(__low2half(h0), __high2half(h0)),
                                                      __hmax(__low2half(h1), __high2half(h1))));
      }
    }
  }
  {  // the block's row maxima
    uint32_t r4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) r4[e] = *reinterpret_cast<const uint32_t*>(&rm[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t other = __shfl_xor_sync(0xffffffffu, r4[e], o);
        const __half2 m = __hmax2(*reinterpret_cast<const __half2*>(&r4[e]),
                                  *reinterpret_cast<const __half2*>(&other));
        r4[e] = *reinterpret_cast<const uint32_t*>(&m);
      }
    if (lane == 0) sh.part[warp] = make_uint4(r4[0], r4[1], r4[2], r4[3]);
  }
  __syncthreads();
  // lane i < 8 of every warp: sx and 1/sx of token i, then shared across the warp
  float sx_l = 0.0f, rcp_l = 0.0f;
  if (lane < kDTok) {
    __half m = __float2half_rn(0.0f);
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) {
      const uint32_t word = (&sh.part[w].x)[lane >> 1];
      const __half2 h2 = *reinterpret_cast<const __half2*>(&word);
      m = __hmax(m, (lane & 1) ? __high2half(h2) : __low2half(h2));
    }
    float mf = __half2float(m);
    if (a.per_tensor)  // one scale for all rows: the largest row absmax (rows past M hold 0)
#pragma unroll
      for (int o = 1; o < kDTok; o <<= 1) mf = fmaxf(mf, __shfl_xor_sync(0x000000FFu, mf, o));
    sx_l = __fdiv_rn(mf, 127.0f);
    rcp_l = mf > 0.0f ? __frcp_rn(sx_l) : 0.0f;
    if (warp == 0) sh.sx[lane] = sx_l;
    if (kTrace && warp == 0 && blockIdx.x == 0 && lane < M && a.trace.sx) a.trace.sx[lane] = sx_l;
  }

  // this warp's k-blocks and the k-steps among them holding an outlier column (bit
  // 4 (kb - kb_begin) + j).  Lane (g, tig) of k-step j of a k-block covers its 8 columns
  // 16 (4 (tig / 2) + j) + 8 (tig % 2) .. + 7 (the chunk 8 (tig / 2) + 2 j + tig % 2), a
  // permutation of the block's 128 columns that both MMA operands follow; with it the 16 lanes
  // of a half-warp read 16 different bank pairs of the swizzled weight rows and of the codes.
  const int kb_begin = warp * KB / kDWarps, kb_end = (warp + 1) * KB / kDWarps;
  const int nsteps = 4 * (kb_end - kb_begin);
  uint32_t ow = 0u;
  if (lane < nsteps) {
    const int kb = kb_begin + lane / 4, j = lane % 4;
    const uint16_t* f2 = reinterpret_cast<const uint16_t*>(sh.flags);
    ow = f2[(kb * 16 + 2 * j) / 2] | f2[(kb * 16 + 8 + 2 * j) / 2];
  }
  const uint32_t outlier_steps = __ballot_sync(0xffffffffu, ow != 0u);
  const int lane_col = 64 * (tig >> 1) + 8 * (tig & 1);  // + 16 j within a k-block

  // ---- int8 codes: xq_s[token][column].  A row with no regular value has 1/sx = 0 and
  // codes 0.
  {
    float sxv[kDTok], rcpv[kDTok];
#pragma unroll
    for (int i = 0; i < kDTok; ++i) {
      sxv[i] = __shfl_sync(0xffffffffu, sx_l, i);
      rcpv[i] = __shfl_sync(0xffffffffu, rcp_l, i);
    }
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const int c = tid + it * kDThreads;
      if (c < chunks) {
#pragma unroll
        for (int i = 0; i < kDTok; ++i) {
          const uint2 q = quantize8(xv[it][i], sxv[i], rcpv[i], xkeep[it]);
          *reinterpret_cast<uint2*>(xq_s + i * xq_ld + c * 8) = q;
          if (kTrace && blockIdx.x == 0 && i < M && a.trace.xq)
            *reinterpret_cast<uint2*>(a.trace.xq + static_cast<size_t>(i) * K + 8 * c) = q;
        }
      }
    }
  }
  __syncthreads();

  // ---- this warp: every tile over k-blocks [kb_begin, kb_end)
  int d[T][2][4];  // two accumulator chains per tile (even and odd k-steps) halve the MMA
                   // dependency chain
  float pf[T][4];
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      d[t][0][e] = d[t][1][e] = 0;
      pf[t][e] = 0.0f;
    }
  bool ok = true;
  if (kb_begin < kb_end) {
    bool landed = true;
    if (lane == 0)
      for (int t = 0; t < T; ++t) landed = landed && mbar_wait_bounded(&sh.full[t], 0, abort);
    ok = __shfl_sync(0xffffffffu, landed ? 1 : 0, 0) != 0;
    for (int t = 0; t < T; ++t) mbar_try_wait(&sh.full[t], 0);  // each lane observes the phase
  }
  if (ok && kb_begin < kb_end) {
    // rows g and g + 8 of the swizzled 16 x 128 tiles: one address per k-step of a k-block
    const uint8_t* wrow[T][4];
#pragma unroll
    for (int t = 0; t < T; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        wrow[t][j] = wt + t * tb + g * 128 + (((4 * (tig >> 1) + j) ^ g) << 4) +
                     (tig & 1) * 8 + kb_begin * (16 * 128);
    const uint8_t* xrow = xq_s + g * xq_ld + lane_col + kb_begin * 128;
    // fp16 term first: the warp's k-steps holding an outlier column, one at a time in a rolled
    // loop (its code exists once); only the outlier columns' activations are nonzero.  Then
    // the int8 k-steps.
    uint32_t rest = outlier_steps;
#pragma unroll 1
    while (rest != 0u) {
      const int st = __ffs(rest) - 1;
      rest &= rest - 1u;
      const int kb = kb_begin + st / 4, j = st % 4;
      const int ch = kb * 16 + 8 * (tig >> 1) + 2 * j + (tig & 1);  // this lane's chunk
      const uint32_t fb = sh.flags[ch];
      uint4 xr = make_uint4(0u, 0u, 0u, 0u);
      if (fb != 0u) {
        const int slot = sh.oslot[ch];
        if (slot < kDOutChunks) xr = sh.xo[slot][g];
        else if (g < M)
          xr = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(g) * K + 8 * ch));
      }
      const uint32_t b0 = mask2(xr.x, fb, 0), b1 = mask2(xr.y, fb, 1);
      const uint32_t b2 = mask2(xr.z, fb, 2), b3 = mask2(xr.w, fb, 3);
      const uint8_t* wb = wt + g * 128 + (((4 * (tig >> 1) + j) ^ g) << 4) + (tig & 1) * 8 +
                          kb * (16 * 128);
#pragma unroll
      for (int t = 0; t < T; ++t) {
        uint32_t ha[2][4];  // rows g, g + 8: fp16 weights of this step's 8 columns
        if (a.W16) {        // the layer's kept fp16 weights
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int n = n0 + 16 * t + 8 * h + g;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (n < N)
              v = __ldg(reinterpret_cast<const uint4*>(
                  a.W16 + static_cast<size_t>(n) * K + kb * 128 + lane_col + 16 * j));
            ha[h][0] = v.x; ha[h][1] = v.y; ha[h][2] = v.z; ha[h][3] = v.w;
          }
        } else {            // fp16(Wq * w_scale) from the resident int8 tile
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint2 w = *reinterpret_cast<const uint2*>(wb + t * tb + 1024 * h);
            ha[h][0] = what2(w.x, 0, swr[t][h]);
            ha[h][1] = what2(w.x, 1, swr[t][h]);
            ha[h][2] = what2(w.y, 0, swr[t][h]);
            ha[h][3] = what2(w.y, 1, swr[t][h]);
          }
        }
        if (kTrace && a.trace.what && fb != 0u) {  // rows g, g + 8, the chunk's outlier columns
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int n = n0 + 16 * t + 8 * h + g;
            if (n >= N) continue;
            unsigned short* dst =
                reinterpret_cast<unsigned short*>(a.trace.what) + static_cast<size_t>(n) * K + 8 * ch;
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if ((fb >> e) & 1u)
                dst[e] = static_cast<unsigned short>(ha[h][e / 2] >> (16 * (e & 1)));
          }
        }
        mma_f16_16816(pf[t], ha[0][0], ha[1][0], ha[0][1], ha[1][1], b0, b1);
        mma_f16_16816(pf[t], ha[0][2], ha[1][2], ha[0][3], ha[1][3], b2, b3);
      }
    }
    for (int kb = kb_begin; kb < kb_end; ++kb) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint2 xb = *reinterpret_cast<const uint2*>(xrow + 16 * j);
        uint2 w[T][2];
#pragma unroll
        for (int t = 0; t < T; ++t) {
          w[t][0] = *reinterpret_cast<const uint2*>(wrow[t][j]);
          w[t][1] = *reinterpret_cast<const uint2*>(wrow[t][j] + 1024);
          mma_s8_16832(d[t][j & 1], w[t][0].x, w[t][1].x, w[t][0].y, w[t][1].y, xb.x, xb.y);
        }
      }
#pragma unroll
      for (int t = 0; t < T; ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j) wrow[t][j] += 16 * 128;
      xrow += 128;
    }
  }
  if (!ok) report(a.status, INT8MM_ERR_TIMEOUT);
  // partial sums into the weight area (every warp is done reading it)
  __syncthreads();
  int32_t* stage_i = reinterpret_cast<int32_t*>(wt);
  float* stage_p = reinterpret_cast<float*>(wt + kDWarps * kDTok * kLd * 4);
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int o = (warp * kDTok + 2 * tig) * kLd + 16 * t + g;
    stage_i[o] = d[t][0][0] + d[t][1][0];
    stage_i[o + kLd] = d[t][0][1] + d[t][1][1];
    stage_i[o + 8] = d[t][0][2] + d[t][1][2];
    stage_i[o + kLd + 8] = d[t][0][3] + d[t][1][3];
    stage_p[o] = pf[t][0];
    stage_p[o + kLd] = pf[t][1];
    stage_p[o + 8] = pf[t][2];
    stage_p[o + kLd + 8] = pf[t][3];
  }
  __syncthreads();
  if (e_live) {  // token ei, channel n0 + ec: the 16 warps in a fixed order
    int32_t acc = 0;
    float P = 0.0f;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) {
      acc += stage_i[(w * kDTok + ei) * kLd + ec];
      P += stage_p[(w * kDTok + ei) * kLd + ec];
    }
    const int n = n0 + ec;
    const float y = static_cast<float>(acc) * sh.sx[ei] * e_sw + P + e_bias;
    a.Y[static_cast<size_t>(ei) * N + n] = __float2half_rn(y);
    if (a.acc) a.acc[static_cast<size_t>(ei) * N + n] = sh.abort ? 0 : acc;
  }
  if (tid == 0) {
    // every copy this CTA started has landed before it exits (normally long ago)
    int dummy = 0;
    for (int t = 0; t < T; ++t) mbar_wait_bounded(&sh.full[t], 0, &dummy);
  }
}

}  // namespace

DecodePlan plan_decode(int M, int N, int K) {
  DecodePlan p = {};
  p.fits = false;
  if (M > kDTok || K % 128 != 0 || K / 128 > kDMaxKb || N <= 0 || M <= 0) return p;
  p.tiles = K <= 4096 ? 2 : 1;
  p.smem = decode_smem_bytes(p.tiles, K);
  p.ctas = (N + 16 * p.tiles - 1) / (16 * p.tiles);
  p.fits = p.smem + sizeof(DecodeShared) <= kDSmemMax;
  return p;
}

cudaError_t launch_decode(const CUtensorMap& map_wq, const DecodeArgs& a, const DecodePlan& p,
                          cudaStream_t stream, bool pdl) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != configured_device) {  // all the shared memory a CTA may have beside the static
    for (const void* k : {reinterpret_cast<const void*>(decode_kernel<2, 1, false>),
                          reinterpret_cast<const void*>(decode_kernel<1, 2, false>),
                          reinterpret_cast<const void*>(decode_kernel<2, 1, true>),
                          reinterpret_cast<const void*>(decode_kernel<1, 2, true>)}) {
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, k);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kDSmemMax - fa.sharedSizeBytes));
      if (e != cudaSuccess) return e;
    }
    configured_device = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ctas);
  cfg.blockDim = dim3(kDThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  // K <= 4096: two tiles, one chunk of X per thread; up to 8192: one tile, two chunks
  const bool trace = a.trace.xq || a.trace.sx || a.trace.flags || a.trace.what;
  if (trace)
    return p.tiles == 2 ? cudaLaunchKernelEx(&cfg, decode_kernel<2, 1, true>, map_wq, a)
                        : cudaLaunchKernelEx(&cfg, decode_kernel<1, 2, true>, map_wq, a);
  return p.tiles == 2 ? cudaLaunchKernelEx(&cfg, decode_kernel<2, 1, false>, map_wq, a)
                      : cudaLaunchKernelEx(&cfg, decode_kernel<1, 2, false>, map_wq, a);
}

}  // namespace i8mm
