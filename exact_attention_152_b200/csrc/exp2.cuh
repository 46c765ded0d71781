// exp2 on the FMA pipe (software), shared by the attention kernel and the
// building-block tests.
#pragma once

namespace eab {

// exp2 on the FMA pipe: 2^x = 2^n * p(f), n = round-to-nearest(x), f = x - n in
// [-1/2, 1/2].  p is a cubic with p(0) = 1 exactly, fitted by this library for
// minimum max relative error (1.01e-4, below BF16's 2^-9 half ulp) -- see
// fit_exp2_poly.py.  n is read out of the low mantissa bits of x + 1.5*2^23
// and added straight into the exponent field.  x is clamped at -127, where the
// result is exactly +0 (so masked scores give weight 0).
constexpr float kExpC1 = 0x1.62f5fap-1f;
constexpr float kExpC2 = 0x1.f00c4cp-3f;
constexpr float kExpC3 = 0x1.c2a216p-5f;

__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -127.0f);
  const float kShift = 12582912.0f;  // 1.5 * 2^23
  const float t = __fadd_rn(x, kShift);
  const float n = __fsub_rn(t, kShift);
  const float f = __fsub_rn(x, n);
  float p = __fmaf_rn(kExpC3, f, kExpC2);
  p = __fmaf_rn(p, f, kExpC1);
  p = __fmaf_rn(p, f, 1.0f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

}  // namespace eab
