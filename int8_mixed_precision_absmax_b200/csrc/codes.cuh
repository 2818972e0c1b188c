// codes.cuh -- the activation quantizer shared by the kernels: the int8 codes rne(RN(x / s)) of
// 8 binary16 values (one 16-byte chunk of a row), x / s being the IEEE float32 quotient.
//
// [P5] "PyTorch 2.9 支持 LLM.int8()", section "LLM.int8() 是怎么做到几乎无损的", item 2:
// codes round(x / s) with s = absmax / 127 per row (or per tensor).
//
// The quotient comes from one correction of x * r, r = RN(1 / s), the method of P. Markstein
// (IBM J. Res. Dev. 34(1), 1990; also his "IA-64 and Elementary Functions", 2000):
//   q0 = RN(x r),  rho = x - q0 s (exact: one FMA),  q1 = RN(q0 + rho r) = RN(x / s).
// On the domain of the activation passes (x and absmax binary16, |x| <= absmax,
// s = RN(absmax / 127)) q1 equals the IEEE quotient for every pair (checked on the GPU for all
// 503,856,639 pairs with x >= 0; the steps are odd in x, but x = -0 gives +0 for -0, the same
// code), and the tests check it on the CPU for sampled scales and the codes on the GPU against
// the oracle.  1.5 * 2^23 + q1 rounded to an integer (ties to even) then holds rne(q1)
// in its low byte in two's complement (1.5 * 2^23 has a zero low byte).  On regular columns
// |q1| <= 127, so no clamp is needed; s = 0 (a row whose regular columns are all 0) comes with
// r = 0 and gives code 0.  Outlier columns may hold any value here: callers mask their bytes.
// Two lanes per packed fp32 operation (mul/fma/add.rn.f32x2, sm_100): each lane is rounded as
// the scalar operation is.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace i8mm {

__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, uint32_t& lo, uint32_t& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// The 8 codes of chunk v, packed little-endian (not masked).
__device__ __forceinline__ uint2 codes8(const uint4& v, float s, float rcp) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const uint64_t r2 = f32x2_pack(rcp, rcp), ns2 = f32x2_pack(-s, -s),
                 k2 = f32x2_pack(kRound, kRound);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t qb[8];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[p]));
    const uint64_t x2 = f32x2_pack(f.x, f.y);
    const uint64_t q0 = f32x2_mul(x2, r2);
    const uint64_t rho = f32x2_fma(q0, ns2, x2);
    const uint64_t q1 = f32x2_fma(rho, r2, q0);
    f32x2_unpack(f32x2_add(q1, k2), qb[2 * p], qb[2 * p + 1]);
  }
  const uint32_t lo = __byte_perm(__byte_perm(qb[0], qb[1], 0x0040), __byte_perm(qb[2], qb[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(qb[4], qb[5], 0x0040), __byte_perm(qb[6], qb[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

// Byte masks that clear the codes of the chunk's outlier columns (bit e set -> byte e = 0).
__device__ __forceinline__ uint2 keep_bytes(uint32_t bits) {
  const uint32_t lo = ~((((bits & 0xFu) * 0x204081u) & 0x01010101u) * 0xFFu);
  const uint32_t hi = ~((((bits >> 4) * 0x204081u) & 0x01010101u) * 0xFFu);
  return make_uint2(lo, hi);
}

}  // namespace i8mm
