// exp2 on the FMA pipe (software), shared by the attention kernel and the
// building-block tests.
#pragma once

#include "sm100.cuh"

namespace eab {

// exp2 on the FMA pipe: 2^x = 2^n * p(f), n = round-to-nearest(x), f = x - n in
// [-1/2, 1/2].  p is a cubic with p(0) = 1 exactly whose other coefficients
// minimise the maximum relative error |p(f)/2^f - 1| on [-1/2, 1/2] (a linear
// program on a dense grid, rounded to fp32; tests/test_exp2_coeffs.py solves
// it again): 1.01e-4, far below BF16's unit roundoff 2^-8.  n is read out of
// the low mantissa bits of x + 1.5*2^23
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

// The same polynomial exp2 on a pair of values with packed fp32 instructions:
// the rounding, the reduction and the Horner steps each cost one instruction
// for both lanes; only the clamp and the exponent insertion stay scalar.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
  x.x = fmaxf(x.x, -127.0f);
  x.y = fmaxf(x.y, -127.0f);
  const float2 kShift = make_float2(12582912.0f, 12582912.0f);
  const float2 t = fadd2(x, kShift);
  const float2 n = fsub2(t, kShift);
  const float2 f = fsub2(x, n);
  float2 p = ffma2(make_float2(kExpC3, kExpC3), f, make_float2(kExpC2, kExpC2));
  p = ffma2(p, f, make_float2(kExpC1, kExpC1));
  p = ffma2(p, f, make_float2(1.0f, 1.0f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

}  // namespace eab
