// gemm.cu -- the tensor-core half of the LLM.int8() layer on sm_100a.
//
// One persistent, warp-specialised kernel computes, per 128 x 256 output tile,
//   A = Xq . Wq^T         int8 x int8 -> int32   tcgen05.mma kind::i8, TMEM accumulator
//   P = X_O . W_hat_O^T   fp16 x fp16 -> fp32    tcgen05.mma kind::f16, second accumulator
// and the fused epilogue Y = fp16(A * sx[i] * w_scale[n] + P + bias[n])
// ([P2] "8位量化实战：离群值处理与显存优化避坑指南" section 2.3: the int8 and fp16 products
// are computed separately and summed; [P5] "PyTorch 2.9 支持 LLM.int8()" item 3: the
// results are merged at the end).  The dequantization by the outer product of the row
// and column scales undoes x ~ q * sx and w ~ q * w_scale of [P5] items 1 and 2.
//
// Roles (320 threads): warp 0 issues TMA loads into a 4-stage shared-memory ring, warp 1
// allocates tensor memory and issues the MMAs (one thread), warps 2-9 drain the
// accumulators (two warps per 32-lane TMEM quadrant, each taking half of the tile's columns;
// the tile's column scales and bias are staged in shared memory once).  With both products
// present the 512 TMEM columns hold one int32 and one fp32 accumulator; with only one of
// them, two accumulator slots alternate so the epilogue of a tile overlaps the next
// tile's main loop.  With both products the epilogue works in two phases: it folds the
// int32 accumulator, the scales, the fp32 outlier term and the bias into fp32 Y written
// back over the outlier accumulator (tcgen05.st) and releases the int32 columns, so the
// next tile's int8 MMAs start at once; it then converts and stores Y and releases the
// fp32 columns, which the next tile needs only for its fp16 MMAs, issued last.
// Every wait is bounded (ptx.cuh); a wait that gives up writes
// INT8MM_ERR_TIMEOUT to the status word, and the block drains its in-flight copies and
// MMAs, frees its tensor memory and exits.
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kStages = 4;
constexpr int kABytes = kBM * kBKBytes;  // 16 KB
constexpr int kBBytes = kBN * kBKBytes;  // 32 KB
constexpr int kThreads = 320;
constexpr int kEpiThreads = kThreads - 64;  // warps 2..9
constexpr uint32_t kTmemCols = 512;


struct GemmShared {
  uint8_t a[kStages][kABytes];
  uint8_t b[kStages][kBBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float wscale[2][kBN];  // the tile's column scales and bias, by accumulator slot parity
  float bias[2][kBN];
};
constexpr size_t kSmemBytes = sizeof(GemmShared) + 1024;  // + alignment slack

// Tiles in groups of gm row tiles: inside a group the row tile varies fastest, so the CTAs
// of one wave share each weight tile through L2 while the group's activation rows (sized by
// the host to stay resident in L2) are reused by every wave of the group.
struct TileSchedule {
  int m_tiles, n_tiles, tiles, gm, bn;
  __device__ void coords(int tile, int& m0, int& n0) const {
    const int per_group = gm * n_tiles;
    const int g = tile / per_group;
    const int first = g * gm;
    const int rows = min(gm, m_tiles - first);
    const int r = tile - g * per_group;
    m0 = (first + r % rows) * kBM;
    n0 = (r / rows) * bn;
  }
};

// Named barrier 1 of the epilogue warps; the second form returns whether any of them
// passed `v` true (one decision for all, so they leave the tile loop together).
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
}
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(kEpiThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_xq, const __grid_constant__ CUtensorMap map_wq,
                const __grid_constant__ CUtensorMap map_xo, const __grid_constant__ CUtensorMap map_wo,
                const GemmArgs args) {
  extern __shared__ uint8_t gemm_smem_raw[];
  GemmShared& S = *reinterpret_cast<GemmShared*>(
      (reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.tmem_full[b], 1);
      mbar_init(&S.tmem_empty[b], kEpiThreads);
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
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // Everything above overlaps the previous kernel; inputs are read only after this.  The next
  // launch may then start its own prologue (it waits for this grid before reading anything).
  grid_dependency_wait();
  grid_launch_dependents();

  const int M = args.M, N = args.N, K = args.K;
  const int n_out = args.n_out ? *args.n_out : 0;
  const int kb_i8 = (n_out >= K) ? 0 : (K + kBKBytes - 1) / kBKBytes;  // Xq == 0 if all outliers
  const int kb_f16 = (n_out + 63) / 64;
  const int kb_total = kb_i8 + kb_f16;
  const bool both = kb_i8 > 0 && kb_f16 > 0;
  const int nslots = both ? 1 : 2;
  const int bn = args.bn > 0 ? args.bn : kBN;  // channels per tile
  const uint32_t idesc_i8 = idesc_i8_s32(kBM, bn);
  const uint32_t idesc_f16 = idesc_f16_f32(kBM, bn);
  TileSchedule sched;
  sched.bn = bn;
  sched.m_tiles = (M + kBM - 1) / kBM;
  sched.n_tiles = (N + bn - 1) / bn;
  sched.tiles = sched.m_tiles * sched.n_tiles;
  sched.gm = (args.group_m > 0 && args.group_m < sched.m_tiles) ? args.group_m : sched.m_tiles;
  const uint32_t tmem = S.tmem_base;
  volatile int* abort = &S.abort;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ producer: TMA into the ring
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < sched.tiles; tile += gridDim.x) {
        int m0, n0;
        sched.coords(tile, m0, n0);
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!mbar_wait_bounded(&S.empty[stage], phase ^ 1u, abort)) { ok = false; break; }
          mbar_arrive_expect_tx(&S.full[stage], kABytes + bn * kBKBytes);
          if (kb < kb_i8) {
            tma_load_2d(&map_xq, S.a[stage], &S.full[stage], kb * kBKBytes, m0);
            tma_load_2d(&map_wq, S.b[stage], &S.full[stage], kb * kBKBytes, n0);
          } else {
            const int k = (kb - kb_i8) * 64;
            tma_load_2d(&map_xo, S.a[stage], &S.full[stage], k, m0);
            tma_load_2d(&map_wo, S.b[stage], &S.full[stage], k, n0);
          }
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // let every issued copy land before the block can exit (bounded, abort ignored)
      int dummy = 0;
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
        mbar_wait_bounded(&S.full[j % kStages], static_cast<uint32_t>(j / kStages) & 1u, &dummy);
      if (!ok) report(args.status, INT8MM_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < sched.tiles; tile += gridDim.x, ++it) {
        const int slot = (nslots == 1) ? 0 : (it & 1);
        const uint32_t use = (nslots == 1) ? it : (it >> 1);
        if (!mbar_wait_bounded(&S.tmem_empty[slot], (use & 1u) ^ 1u, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_i8 = tmem + (both ? 0u : slot * 256u);
        const uint32_t d_f32 = tmem + (both ? 256u : slot * 256u);
        for (int kb = 0; kb < kb_total; ++kb) {
          if (both && kb == kb_i8) {  // the fp32 columns: free once the last tile's Y is out
            if (!mbar_wait_bounded(&S.tmem_empty[1], (static_cast<uint32_t>(it) & 1u) ^ 1u,
                                   abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (!mbar_wait_bounded(&S.full[stage], phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_addr(S.a[stage]);
          const uint32_t b0 = smem_addr(S.b[stage]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 4 x 32 bytes along K per stage
            const uint64_t ad = sw128_kmajor_desc(a0 + 32u * k);
            const uint64_t bd = sw128_kmajor_desc(b0 + 32u * k);
            if (kb < kb_i8)
              mma_i8(d_i8, ad, bd, idesc_i8, (kb > 0 || k > 0) ? 1u : 0u);
            else
              mma_f16(d_f32, ad, bd, idesc_f16, (kb > kb_i8 || k > 0) ? 1u : 0u);
          }
          mma_commit(&S.empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&S.tmem_full[slot]);
      }
      // every MMA issued so far must finish before tensor memory is freed
      mma_commit(&S.drain);
      int dummy = 0;
      mbar_wait_bounded(&S.drain, 0, &dummy);
      if (!ok) report(args.status, INT8MM_ERR_TIMEOUT);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..9)
    const int quad = warp & 3;                // TMEM lanes 32 quad .. 32 quad + 31
    const int half = (warp - 2) / 4;          // the first or the second half of the tile's columns
    // 16-column chunks: the first half takes ceil(chunks / 2) of them
    const int c_split = (bn / 16 + 1) / 2 * 16;
    const int c_begin = half ? c_split : 0, c_end = half ? bn : c_split;
    const int et = threadIdx.x - 64;          // 0 .. kEpiThreads - 1
    const bool vec_ok = (N % 8) == 0;
    int it = 0;
    for (int tile = blockIdx.x; tile < sched.tiles; tile += gridDim.x, ++it) {
      const int slot = (nslots == 1) ? 0 : (it & 1);
      const uint32_t use = (nslots == 1) ? it : (it >> 1);
      int m0, n0;
      sched.coords(tile, m0, n0);
      // the tile's column scales and bias (buffer it & 1: the previous tile's may still be
      // in use by a slower epilogue warp)
      {
        const int n = n0 + et;
        // (the raw int32 product has neither: w_scale and bias are null there)
        S.wscale[it & 1][et] = (et < bn && n < N && args.w_scale) ? args.w_scale[n] : 0.0f;
        S.bias[it & 1][et] = (et < bn && n < N && args.bias) ? __half2float(args.bias[n]) : 0.0f;
        epi_sync();
      }
      const bool landed = mbar_wait_bounded(&S.tmem_full[slot], use & 1u, abort);
      if (epi_any(!landed)) {  // every epilogue thread takes the same branch
        report(args.status, INT8MM_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int row = m0 + quad * 32 + lane;
      const bool row_ok = row < M;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
      const uint32_t t_i8 = lane_base + (both ? 0u : slot * 256u);
      const uint32_t t_f32 = lane_base + (both ? 256u : slot * 256u);
      const float sx = (args.Y && row_ok) ? args.xscale[row] : 0.0f;
      const float* wsc = S.wscale[it & 1];
      const float* bsc = S.bias[it & 1];
      if (both) {
        // phase 1: Y in fp32 over the outlier accumulator, then the int32 columns are free
        for (int c = c_begin; c < c_end; c += 16) {
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
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 ws = *reinterpret_cast<const float4*>(wsc + c + 4 * j4);
            const float4 bs = *reinterpret_cast<const float4*>(bsc + c + 4 * j4);
            const float wv[4] = {ws.x, ws.y, ws.z, ws.w}, bv[4] = {bs.x, bs.y, bs.z, bs.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 4 * j4 + e;
              const float acc = static_cast<float>(static_cast<int32_t>(ra[j])) * sx * wv[e] +
                                __uint_as_float(rp[j]);
              rp[j] = __float_as_uint(acc + bv[e]);
            }
          }
          tmem_st16(t_f32 + c, rp);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&S.tmem_empty[0]);
        // phase 2: Y out, then the fp32 columns are free
        for (int c = c_begin; c < c_end; c += 16) {
          uint32_t ry[16];
          __syncwarp();
          tmem_ld16(t_f32 + c, ry);
          tmem_ld_wait();
          const int n = n0 + c;
          const int valid = min(16, N - n);
          if (row_ok && valid > 0 && args.Y) {
            __half* dst = args.Y + static_cast<size_t>(row) * N + n;
            if (vec_ok && valid == 16) {
              uint32_t w[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const __half2 h = __floats2half2_rn(__uint_as_float(ry[2 * e]),
                                                    __uint_as_float(ry[2 * e + 1]));
                w[e] = *reinterpret_cast<const uint32_t*>(&h);
              }
              reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
              reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (j < valid) dst[j] = __float2half_rn(__uint_as_float(ry[j]));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&S.tmem_empty[1]);
        continue;
      }
      for (int c = c_begin; c < c_end; c += 16) {
        uint32_t ra[16], rp[16];
        __syncwarp();  // the tensor-memory loads are warp-collective
        if (kb_i8 > 0) tmem_ld16(t_i8 + c, ra);
        if (kb_f16 > 0) tmem_ld16(t_f32 + c, rp);
        tmem_ld_wait();
        const int n = n0 + c;
        const int valid = min(16, N - n);
        if (row_ok && valid > 0 && args.C) {
          int32_t* dst = args.C + static_cast<size_t>(row) * N + n;
          if (valid == 16 && (N % 4) == 0) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              reinterpret_cast<int4*>(dst)[v] =
                  make_int4(kb_i8 ? ra[4 * v] : 0, kb_i8 ? ra[4 * v + 1] : 0,
                            kb_i8 ? ra[4 * v + 2] : 0, kb_i8 ? ra[4 * v + 3] : 0);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j < valid) dst[j] = kb_i8 ? static_cast<int32_t>(ra[j]) : 0;
          }
        }
        if (row_ok && valid > 0 && args.Y) {
          float y[16];
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 ws = *reinterpret_cast<const float4*>(wsc + c + 4 * j4);
            const float4 bs = *reinterpret_cast<const float4*>(bsc + c + 4 * j4);
            const float wv[4] = {ws.x, ws.y, ws.z, ws.w}, bv[4] = {bs.x, bs.y, bs.z, bs.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 4 * j4 + e;
              float acc = 0.0f;
              if (kb_i8 > 0) acc = static_cast<float>(static_cast<int32_t>(ra[j])) * sx * wv[e];
              if (kb_f16 > 0) acc += __uint_as_float(rp[j]);
              y[j] = acc + bv[e];
            }
          }
          __half* dst = args.Y + static_cast<size_t>(row) * N + n;
          if (vec_ok && valid == 16) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const __half2 h = __floats2half2_rn(y[2 * e], y[2 * e + 1]);
              w[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j < valid) dst[j] = __float2half_rn(y[j]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&S.tmem_empty[slot]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

namespace {

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn tmap_encoder() {
  static EncodeFn encode = nullptr;
  if (encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return nullptr;
    encode = reinterpret_cast<EncodeFn>(fn);
  }
  return encode;
}

}  // namespace

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                    uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                    uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  EncodeFn encode = tmap_encoder();
  if (!encode) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t elem_strides[2] = {1, 1};
  return encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                    const uint64_t (&dims)[3], const uint64_t (&strides_bytes)[2],
                    const uint32_t (&box)[3], CUtensorMapSwizzle swizzle) {
  EncodeFn encode = tmap_encoder();
  if (!encode) return false;
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  return encode(map, dtype, 3, const_cast<void*>(base), d, st, bx, elem_strides,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gemm_tile_width(int M, int N) {
  // Measured: the widths that fill the last wave (224 for the 13B-shaped layer, 240 for
  // prefill up_proj) ran 10% faster in an isolated launch of the 13B-shaped layer and within 1%
  // under steps back to back at the 1 kW power cap (where a partly filled last wave costs
  // less: the idle SMs let the busy ones clock higher).
  const int ctas = device_sm_count();
  const long long m_tiles = (M + kBM - 1) / kBM;
  constexpr int kFixed = 32;  // per-tile cost beyond the MMA columns, in the same units
  int best = kBN;
  long long best_cost = -1;
  for (int bn = kBN; bn >= 128; bn -= 16) {
    const long long tiles = m_tiles * ((N + bn - 1) / bn);
    const long long waves = (tiles + ctas - 1) / ctas;
    const long long cost = waves * (bn + kFixed);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

cudaError_t launch_gemm(const GemmMaps& maps, const GemmArgs& a, cudaStream_t stream, bool pdl) {
  static int configured_device = -1;
  static int num_sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  const int m_tiles = (a.M + kBM - 1) / kBM;
  const int bn = a.bn > 0 ? a.bn : kBN;
  const int tiles = m_tiles * ((a.N + bn - 1) / bn);
  // row tiles per group: as many as keep the group's int8 activations (gm x 128 rows x K
  // bytes) within 32 MiB of L2, balanced over the groups
  GemmArgs args = a;
  const long long budget = 32ll << 20;
  const long long row_tile_bytes = static_cast<long long>(kBM) * a.K;
  const int gm_max = static_cast<int>(budget / row_tile_bytes) > 1
                         ? static_cast<int>(budget / row_tile_bytes) : 1;
  const int groups = (m_tiles + gm_max - 1) / gm_max;
  args.group_m = (m_tiles + groups - 1) / groups;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles < num_sms ? tiles : num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_kernel, maps.xq, maps.wq, maps.xo, maps.wo, args);
}

}  // namespace i8mm
