// 2^x evaluated on the FMA and integer pipes, for two values at once.
//
// The attention softmax needs one exponential per score; the special-function
// unit (MUFU ex2) alone cannot keep up with the tcgen05 tensor pipe, so part of
// the exponentials are computed here instead.
//
// Method (range reduction in the style of Cody and Waite, then a polynomial):
//   x  is clamped to [-126, +inf) so that 2^j below stays a normal number;
//   t  = x + 1.5*2^23 rounds x to the nearest integer j in t's low mantissa bits;
//   j  = t - 1.5*2^23 (exact), f = x - j in [-1/2, 1/2];
//   2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 (Horner, fused multiply-adds);
//   2^x = 2^f * 2^j, formed by adding j to the exponent field: the low bits of
//   t's encoding are 0x4B400000 + j, and (0x4B400000 << 23) vanishes mod 2^32,
//   so bits(t) << 23 == j << 23.
// The cubic is this library's own minimax fit of the relative error of 2^f on
// [-1/2, 1/2] (csrc/fit_exp2_poly.py, Lawson iteration): max relative error
// 7.5e-5 in fp32, below the bf16 rounding (2^-9) that P goes through anyway.
// Valid for x <= 127; inputs below -126 return 2^-126 (≈ 1.2e-38) instead of a
// smaller number, which callers must tolerate (a softmax row sum is >= 1).
#pragma once

#include <cuda_runtime.h>

namespace tessera {

struct Exp2Poly {
  static constexpr float c0 = 0.9999280571937561f;
  static constexpr float c1 = 0.6932609677314758f;
  static constexpr float c2 = 0.2426111251115799f;
  static constexpr float c3 = 0.0551716685295105f;
  static constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  static constexpr float kMin = -126.0f;
};

__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, Exp2Poly::kMin);
  x.y = fmaxf(x.y, Exp2Poly::kMin);
  const float2 t = __fadd2_rn(x, make_float2(Exp2Poly::kRound, Exp2Poly::kRound));
  const float2 j = __fadd2_rn(t, make_float2(-Exp2Poly::kRound, -Exp2Poly::kRound));
  const float2 f = __ffma2_rn(j, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(make_float2(Exp2Poly::c3, Exp2Poly::c3), f,
                        make_float2(Exp2Poly::c2, Exp2Poly::c2));
  p = __ffma2_rn(p, f, make_float2(Exp2Poly::c1, Exp2Poly::c1));
  p = __ffma2_rn(p, f, make_float2(Exp2Poly::c0, Exp2Poly::c0));
  float2 r;
  r.x = __uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23));
  r.y = __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23));
  return r;
}

}  // namespace tessera
