// gemm2.cu -- the tensor-core half of the LLM.int8() layer for many rows, one 256 x 256 output
// tile per pair of CTAs (tcgen05 cta_group::2).
//
// Per pair tile it computes what gemm.cu computes per 128 x 256 tile,
//   A = Xq . Wq^T         int8 x int8 -> int32   tcgen05.mma kind::i8
//   P = X_O . W_hat_O^T   fp16 x fp16 -> fp32    tcgen05.mma kind::f16
//   Y = fp16(A * sx[i] * w_scale[n] + P + bias[n])
// ([P2] "8位量化实战：离群值处理与显存优化避坑指南" section 2.3: the two products computed
// apart and summed; [P5] "PyTorch 2.9 支持 LLM.int8()" items 1-3: the outer product of the
// row and column scales undoes the quantization, the results are merged at the end).
//
// The two CTAs of a 2-CTA cluster share each tile: per 128-byte k-block each loads 128 rows of
// the activation operand and 128 output channels of the weight operand into its own shared
// memory (16 + 16 KB per stage, a 6-stage ring), and one thread of the even-ranked CTA (the
// leader) issues an MMA of M = 256 rows x N = 256 channels that reads the operands of both; the
// accumulator lands in both CTAs' tensor memory, 128 rows each.  For the same multiply-adds an
// SM fetches 32 instead of 48 KB per k-block than with one CTA per 128 x 256 tile, so the same
// shared memory keeps 1.5 times as much of the operand stream in flight.  That matters because
// the ring is latency-bound: a stage is locked from its load until about 1700 cycles after its
// MMAs finish (when their commit reaches the producer), so the tensor pipe only stays busy when
// the ring holds more MMA work than load latency plus that round trip.  (Measured: 4, 6 and 7
// stages ran within 1% of each other, and asking L2 for each stage's boxes eight k-blocks ahead
// of its loads doubled the L2 requests and slowed the kernel by a fifth.)  The epilogue reads the
// column scales from global memory (L1) and leaves the shared memory to the ring.
//
// Roles (320 threads per CTA): warp 0 issues TMA loads (both CTAs; completion is counted on
// the leader's barrier), warp 1 allocates tensor memory (both CTAs, together) and issues the
// MMAs (leader only), warps 2-9 drain this CTA's 128 accumulator rows exactly as in gemm.cu,
// and release a slot by arriving on the leader's barrier.  Every wait is bounded (ptx.cuh).
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kPM = 256;                             // rows of a pair tile (128 per CTA)
constexpr int kPN = 256;                             // output channels of a pair tile
constexpr int kHalfRows = 128;                       // operand rows one CTA holds
constexpr int kPStages = 6;
constexpr int kOpBytes = kHalfRows * kBKBytes;       // 16 KB: 128 rows x 128 bytes
constexpr int kPThreads = 320;
constexpr int kPEpiThreads = kPThreads - 64;         // warps 2..9
constexpr int kPEpiWarps = kPEpiThreads / 32;
constexpr uint32_t kPTmemCols = 512;
constexpr uint32_t kPIdescI8 = idesc_i8_s32(kPM, kPN);
constexpr uint32_t kPIdescF16 = idesc_f16_f32(kPM, kPN);

struct PairShared {
  uint8_t a[kPStages][kOpBytes];  // this CTA's 128 activation rows of each stage
  uint8_t b[kPStages][kOpBytes];  // this CTA's 128 weight rows (output channels)
  uint64_t full[kPStages];        // leader: both CTAs' operands of a stage have landed
  uint64_t empty[kPStages];       // both: the pair's MMAs are done with a stage
  uint64_t tmem_full[2];          // both: an accumulator slot holds a finished tile
  uint64_t tmem_empty[2];         // leader: the epilogues of both CTAs are done with a slot
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kPSmemBytes = sizeof(PairShared) + 1024;  // + alignment slack

// Pair tiles in groups of gm row tiles, the row tile fastest inside a group (see gemm.cu).
struct PairSchedule {
  int m_tiles, n_tiles, tiles, gm;
  __device__ void coords(int tile, int& m0, int& n0) const {
    const int per_group = gm * n_tiles;
    const int g = tile / per_group;
    const int first = g * gm;
    const int rows = min(gm, m_tiles - first);
    const int r = tile - g * per_group;
    m0 = (first + r % rows) * kPM;
    n0 = (r / rows) * kPN;
  }
};

__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(kPEpiThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// Column scales and bias of the 16 output channels n .. n + 15 (`valid` of them inside N).
__device__ __forceinline__ void load_col_params(const GemmArgs& args, int n, int valid,
                                                float (&wv)[16], float (&bv)[16]) {
  if (valid >= 16) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const float4 w = __ldg(reinterpret_cast<const float4*>(args.w_scale + n) + v);
      wv[4 * v] = w.x; wv[4 * v + 1] = w.y; wv[4 * v + 2] = w.z; wv[4 * v + 3] = w.w;
    }
    if (args.bias) {
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const uint4 h = __ldg(reinterpret_cast<const uint4*>(args.bias + n) + v);
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hw[e]));
          bv[8 * v + 2 * e] = f.x;
          bv[8 * v + 2 * e + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) bv[j] = 0.0f;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      wv[j] = j < valid ? args.w_scale[n + j] : 0.0f;
      bv[j] = (j < valid && args.bias) ? __half2float(args.bias[n + j]) : 0.0f;
    }
  }
}

// This warp is done with its tensor-memory columns: tell the leader's MMA thread.
__device__ __forceinline__ void release_slot(uint32_t bar_cluster, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(bar_cluster);
}

}  // namespace

__global__ void __launch_bounds__(kPThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap map_xq,
                     const __grid_constant__ CUtensorMap map_wq,
                     const __grid_constant__ CUtensorMap map_xo,
                     const __grid_constant__ CUtensorMap map_wo, const GemmArgs args) {
  extern __shared__ uint8_t pair_smem_raw[];
  PairShared& S = *reinterpret_cast<PairShared*>(
      (reinterpret_cast<uintptr_t>(pair_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0: the leader, 1: its peer
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.tmem_full[b], 1);
      mbar_init(&S.tmem_empty[b], 2 * kPEpiWarps);
    }
    mbar_init(&S.drain, 1);
    S.abort = 0;
    fence_mbarrier_init();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&map_xq);
    prefetch_tmap(&map_wq);
    prefetch_tmap(&map_xo);
    prefetch_tmap(&map_wo);
  }
  if (warp == 1) {
    tmem_alloc_pair(&S.tmem_base, kPTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_barrier_sync();  // both CTAs: barriers initialised, tensor memory allocated
  tc_fence_after();

  // Everything above overlaps the previous kernel; inputs are read only after this.
  grid_dependency_wait();
  grid_launch_dependents();

  const int M = args.M, N = args.N, K = args.K;
  const int n_out = args.n_out ? *args.n_out : 0;
  const int kb_i8 = (n_out >= K) ? 0 : (K + kBKBytes - 1) / kBKBytes;  // Xq == 0 if all outliers
  const int kb_f16 = (n_out + 63) / 64;
  const int kb_total = kb_i8 + kb_f16;
  const bool both = kb_i8 > 0 && kb_f16 > 0;
  const int nslots = both ? 1 : 2;
  PairSchedule sched;
  sched.m_tiles = (M + kPM - 1) / kPM;
  sched.n_tiles = (N + kPN - 1) / kPN;
  sched.tiles = sched.m_tiles * sched.n_tiles;
  sched.gm = (args.group_m > 0 && args.group_m < sched.m_tiles) ? args.group_m : sched.m_tiles;
  const int pair = blockIdx.x / 2, pairs = gridDim.x / 2;
  const int row_off = static_cast<int>(rank) * kHalfRows;
  const uint32_t tmem = S.tmem_base;
  volatile int* abort = &S.abort;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ producer (both CTAs)
      const uint32_t full0 = mapa_shared(smem_addr(&S.full[0]), 0);  // the leader's barriers
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < sched.tiles; tile += pairs) {
        int m0, n0;
        sched.coords(tile, m0, n0);
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!mbar_wait_bounded(&S.empty[stage], phase ^ 1u, abort)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&S.full[stage], 4 * kOpBytes);  // both CTAs' A + B
          const uint32_t fb = full0 + static_cast<uint32_t>(stage * sizeof(uint64_t));
          if (kb < kb_i8) {
            tma_load_2d_pair(&map_xq, S.a[stage], fb, kb * kBKBytes, m0 + row_off);
            tma_load_2d_pair(&map_wq, S.b[stage], fb, kb * kBKBytes, n0 + row_off);
          } else {
            const int k = (kb - kb_i8) * 64;
            tma_load_2d_pair(&map_xo, S.a[stage], fb, k, m0 + row_off);
            tma_load_2d_pair(&map_wo, S.b[stage], fb, k, n0 + row_off);
          }
          ++issued;
          if (++stage == kPStages) { stage = 0; phase ^= 1u; }
        }
      }
      // every issued copy has landed before the block can exit (bounded, abort ignored): the
      // leader sees both CTAs' bytes on its full barriers; the peer sees the MMAs that read its
      // last stage finish
      int dummy = 0;
      if (leader) {
        for (int j = issued > kPStages ? issued - kPStages : 0; j < issued; ++j)
          mbar_wait_bounded_cluster(&S.full[j % kPStages], static_cast<uint32_t>(j / kPStages) & 1u,
                                    &dummy);
      } else if (issued > 0) {
        const int j = issued - 1;
        mbar_wait_bounded(&S.empty[j % kPStages], static_cast<uint32_t>(j / kPStages) & 1u, &dummy);
      }
      if (!ok) report(args.status, INT8MM_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ------------------------------------------------ MMA issuer (leader only)
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < sched.tiles; tile += pairs, ++it) {
        const int slot = (nslots == 1) ? 0 : (it & 1);
        const uint32_t use = (nslots == 1) ? it : (it >> 1);
        if (!mbar_wait_bounded_cluster(&S.tmem_empty[slot], (use & 1u) ^ 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_i8 = tmem + (both ? 0u : slot * 256u);
        const uint32_t d_f32 = tmem + (both ? 256u : slot * 256u);
        for (int kb = 0; kb < kb_total; ++kb) {
          if (both && kb == kb_i8) {  // the fp32 columns: free once the last tile's Y is out
            if (!mbar_wait_bounded_cluster(&S.tmem_empty[1],
                                           (static_cast<uint32_t>(it) & 1u) ^ 1u, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (!mbar_wait_bounded_cluster(&S.full[stage], phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_addr(S.a[stage]);
          const uint32_t b0 = smem_addr(S.b[stage]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 4 x 32 bytes along K per stage
            const uint64_t ad = sw128_kmajor_desc(a0 + 32u * k);
            const uint64_t bd = sw128_kmajor_desc(b0 + 32u * k);
            if (kb < kb_i8)
              mma_pair_i8(d_i8, ad, bd, kPIdescI8, (kb > 0 || k > 0) ? 1u : 0u);
            else
              mma_pair_f16(d_f32, ad, bd, kPIdescF16, (kb > kb_i8 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(&S.empty[stage]);  // frees the stage in both CTAs
          if (++stage == kPStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair(&S.tmem_full[slot]);
      }
      // every MMA issued so far must finish before tensor memory is freed
      mma_commit_pair(&S.drain);
      int dummy = 0;
      mbar_wait_bounded(&S.drain, 0, &dummy);
      if (!ok) report(args.status, INT8MM_ERR_TIMEOUT);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..9, both CTAs)
    const int quad = warp & 3;                // TMEM lanes 32 quad .. 32 quad + 31
    const int half = (warp - 2) / 4;          // columns 128 half .. 128 half + 127
    const bool vec_ok = (N % 8) == 0;
    const uint32_t empty0 = mapa_shared(smem_addr(&S.tmem_empty[0]), 0);
    const uint32_t empty1 = mapa_shared(smem_addr(&S.tmem_empty[1]), 0);
    int it = 0;
    for (int tile = pair; tile < sched.tiles; tile += pairs, ++it) {
      const int slot = (nslots == 1) ? 0 : (it & 1);
      const uint32_t use = (nslots == 1) ? it : (it >> 1);
      int m0, n0;
      sched.coords(tile, m0, n0);
      const bool landed = mbar_wait_bounded(&S.tmem_full[slot], use & 1u, abort);
      if (epi_any(!landed)) {  // every epilogue thread takes the same branch
        report(args.status, INT8MM_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int row = m0 + row_off + quad * 32 + lane;
      const bool row_ok = row < M;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
      const uint32_t t_i8 = lane_base + (both ? 0u : slot * 256u);
      const uint32_t t_f32 = lane_base + (both ? 256u : slot * 256u);
      const float sx = (args.Y && row_ok) ? args.xscale[row] : 0.0f;
      if (both) {
        // phase 1: Y in fp32 over the outlier accumulator, then the int32 columns are free
        for (int c = half * (kPN / 2); c < (half + 1) * (kPN / 2); c += 16) {
          uint32_t ra[16], rp[16];
          __syncwarp();
          tmem_ld16(t_i8 + c, ra);
          tmem_ld16(t_f32 + c, rp);
          tmem_ld_wait();
          const int n = n0 + c;
          const int valid = min(16, N - n);
          if (row_ok && valid > 0 && args.C) {
            int32_t* dst = args.C + static_cast<size_t>(row) * N + n;
            if (valid == 16 && (N % 4) == 0) {
#pragma unroll
              for (int v = 0; v < 4; ++v)
                reinterpret_cast<int4*>(dst)[v] =
                    make_int4(ra[4 * v], ra[4 * v + 1], ra[4 * v + 2], ra[4 * v + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (j < valid) dst[j] = static_cast<int32_t>(ra[j]);
            }
          }
          if (args.Y && valid > 0) {
            float wv[16], bv[16];
            load_col_params(args, n, valid, wv, bv);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float acc = static_cast<float>(static_cast<int32_t>(ra[j])) * sx * wv[j] +
                                __uint_as_float(rp[j]);
              rp[j] = __float_as_uint(acc + bv[j]);
            }
          }
          tmem_st16(t_f32 + c, rp);
        }
        tmem_st_wait();
        release_slot(empty0, lane);
        // phase 2: Y out, 32 columns per load so that each lane writes 64 contiguous bytes of
        // its row (two whole sectors); then the fp32 columns are free
        for (int c = half * (kPN / 2); c < (half + 1) * (kPN / 2); c += 32) {
          uint32_t ry[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_f32 + c, ry);
          tmem_ld_wait();
          const int n = n0 + c;
          const int valid = min(32, N - n);
          if (row_ok && valid > 0 && args.Y) {
            __half* dst = args.Y + static_cast<size_t>(row) * N + n;
            if (vec_ok && valid == 32) {
              uint32_t w[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const __half2 h = __floats2half2_rn(__uint_as_float(ry[2 * e]),
                                                    __uint_as_float(ry[2 * e + 1]));
                w[e] = *reinterpret_cast<const uint32_t*>(&h);
              }
#pragma unroll
              for (int v = 0; v < 4; ++v)
                reinterpret_cast<uint4*>(dst)[v] =
                    make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < valid) dst[j] = __float2half_rn(__uint_as_float(ry[j]));
            }
          }
        }
        release_slot(empty1, lane);
        continue;
      }
      // 32 columns per load: each lane writes 64 contiguous bytes of Y (128 of C) in its row
      for (int c = half * (kPN / 2); c < (half + 1) * (kPN / 2); c += 32) {
        uint32_t ra[32], rp[32];
        __syncwarp();  // the tensor-memory loads are warp-collective
        if (kb_i8 > 0) tmem_ld_32x32b_x32(t_i8 + c, ra);
        if (kb_f16 > 0) tmem_ld_32x32b_x32(t_f32 + c, rp);
        tmem_ld_wait();
        const int n = n0 + c;
        const int valid = min(32, N - n);
        if (row_ok && valid > 0 && args.C) {
          int32_t* dst = args.C + static_cast<size_t>(row) * N + n;
          if (valid == 32 && (N % 4) == 0) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              reinterpret_cast<int4*>(dst)[v] =
                  make_int4(kb_i8 ? ra[4 * v] : 0, kb_i8 ? ra[4 * v + 1] : 0,
                            kb_i8 ? ra[4 * v + 2] : 0, kb_i8 ? ra[4 * v + 3] : 0);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < valid) dst[j] = kb_i8 ? static_cast<int32_t>(ra[j]) : 0;
          }
        }
        if (row_ok && valid > 0 && args.Y) {
          uint32_t w[16];  // Y of the 32 columns as half2 words
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float wv[16], bv[16];
            load_col_params(args, n + 16 * h, min(16, valid - 16 * h), wv, bv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float y2[2];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const int j = 16 * h + 2 * e + q;
                float acc = 0.0f;
                if (kb_i8 > 0)
                  acc = static_cast<float>(static_cast<int32_t>(ra[j])) * sx * wv[2 * e + q];
                if (kb_f16 > 0) acc += __uint_as_float(rp[j]);
                y2[q] = acc + bv[2 * e + q];
              }
              const __half2 hv = __floats2half2_rn(y2[0], y2[1]);
              w[8 * h + e] = *reinterpret_cast<const uint32_t*>(&hv);
            }
          }
          __half* dst = args.Y + static_cast<size_t>(row) * N + n;
          if (vec_ok && valid == 32) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              reinterpret_cast<uint4*>(dst)[v] =
                  make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < valid)
                dst[j] = __ushort_as_half(static_cast<unsigned short>(w[j / 2] >> (16 * (j & 1))));
          }
        }
      }
      release_slot(slot == 0 ? empty0 : empty1, lane);
    }
  }

  // Both CTAs: every MMA is done (the leader drained them), every tensor-memory read and every
  // arrival on the other CTA's barriers has happened; then the pair frees its tensor memory.
  tc_fence_before();
  __syncthreads();
  cluster_barrier_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kPTmemCols);
  }
}

// ------------------------------------------------------------------ host side

cudaError_t launch_gemm_pair(const GemmMaps& maps, const GemmArgs& a, cudaStream_t stream,
                             bool pdl) {
  static int configured_device = -1;
  static int max_pairs = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kPSmemBytes));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2);
    q.blockDim = dim3(kPThreads);
    q.dynamicSmemBytes = kPSmemBytes;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel, &q) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = device_sm_count() / 2;
    }
    max_pairs = n;
    configured_device = dev;
  }
  const int m_tiles = (a.M + kPM - 1) / kPM;
  const int tiles = m_tiles * ((a.N + kPN - 1) / kPN);
  // row tiles per group: as many as keep the group's int8 activations (gm x 256 rows x K
  // bytes) within 32 MiB of L2, balanced over the groups
  GemmArgs args = a;
  const long long budget = 32ll << 20;
  const long long row_tile_bytes = static_cast<long long>(kPM) * a.K;
  const int gm_max = static_cast<int>(budget / row_tile_bytes) > 1
                         ? static_cast<int>(budget / row_tile_bytes) : 1;
  const int groups = (m_tiles + gm_max - 1) / gm_max;
  args.group_m = (m_tiles + groups - 1) / groups;
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = kPSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel, maps.xq, maps.wq, maps.xo, maps.wo, args);
}

}  // namespace i8mm
