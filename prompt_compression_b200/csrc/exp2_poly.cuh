// exp2_poly.cuh -- 2^t on the FMA pipe, two lanes at a time (packed fp32x2).
//
// The scoring epilogues need one exponential per logit per pass; the MUFU
// unit delivers 16 per clock per SM, the FMA pipe 128 fp32 FMAs.  Evaluating
// part of the exponentials here keeps both pipes busy.
//
// Method (range reduction + minimax polynomial):
//   t is clamped to >= -126 (below that 2^t is under the normal range and
//   contributes nothing to the sums it feeds);
//   r = t + 1.5*2^23 rounds t to the nearest integer j in r's low mantissa
//   bits; j = r - 1.5*2^23 exactly; f = t - j lies in [-1/2, 1/2];
//   2^f ~= p(f), p of degree 4 with coefficients from a Remez fit of the
//   relative error on [-1/2, 1/2] (csrc/fit_exp2.py: max relative error
//   2.6e-6 exact, 2.7e-6 evaluated in fp32 Horner form);
//   2^t = p(f) * 2^j is formed by adding j to p's exponent field: the low 9
//   bits of r's bit pattern are j, so (bits(r) << 23) adds j << 23 (mod 2^32).
// Per pair: 2 clamps, 3 range-reduction and 4 Horner fp32x2 operations,
// 2 shift-adds: 11 instructions for 2 exponentials.
#pragma once

#include <cuda_runtime.h>

namespace spk {

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// Remez coefficients c0..c4 of p(f) ~= 2^f (fp32 bit patterns).
#define SPK_EXP2_C0 __uint_as_float(0x3f7ffff4u)
#define SPK_EXP2_C1 __uint_as_float(0x3f31706eu)
#define SPK_EXP2_C2 __uint_as_float(0x3e76036du)
#define SPK_EXP2_C3 __uint_as_float(0x3d650a20u)
#define SPK_EXP2_C4 __uint_as_float(0x3c1ccbebu)

__device__ __forceinline__ float2 exp2_fma_pair(float2 t) {
  t.x = fmaxf(t.x, -126.f);
  t.y = fmaxf(t.y, -126.f);
  const float kRound = 12582912.f;   // 1.5 * 2^23
  const float2 r = __fadd2_rn(t, f2(kRound, kRound));
  const float2 j = __fadd2_rn(r, f2(-kRound, -kRound));
  const float2 f = __ffma2_rn(j, f2(-1.f, -1.f), t);
  float2 p = __ffma2_rn(f2(SPK_EXP2_C4, SPK_EXP2_C4), f, f2(SPK_EXP2_C3, SPK_EXP2_C3));
  p = __ffma2_rn(p, f, f2(SPK_EXP2_C2, SPK_EXP2_C2));
  p = __ffma2_rn(p, f, f2(SPK_EXP2_C1, SPK_EXP2_C1));
  p = __ffma2_rn(p, f, f2(SPK_EXP2_C0, SPK_EXP2_C0));
  return f2(__int_as_float(__float_as_int(p.x) + (__float_as_int(r.x) << 23)),
            __int_as_float(__float_as_int(p.y) + (__float_as_int(r.y) << 23)));
}

__device__ __forceinline__ float2 exp2_mufu_pair(float2 t) {
  float a, b;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(a) : "f"(t.x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(b) : "f"(t.y));
  return f2(a, b);
}

}  // namespace spk
