// exp2_poly.cuh -- 2^x on the FMA pipe, to relieve the MUFU unit.
// Cody-Waite range reduction (n = round(x) through the 1.5 * 2^23 shifter,
// f = x - n in [-1/2, 1/2]) and a cubic p(f) ~ 2^f with minimax relative
// error, coefficients from fit_exp2_poly.py (Lawson iteration); the result
// is p(f) with n added to its exponent field.  Max relative error 7.48e-05
// for x <= 125; inputs below -125 (-inf included) are clamped to -125,
// giving 2^-125 rather than 0, so masked entries must not come here.
#pragma once
#include <stdint.h>
namespace sdpa {
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;  // 1.5 * 2^23: low bits of t hold round(x)
  const float n = t - 12582912.0f;
  const float f = x - n;
  float p = 5.517149344e-02f;
  p = fmaf(p, f, 2.426109314e-01f);
  p = fmaf(p, f, 6.932609677e-01f);
  p = fmaf(p, f, 9.999280572e-01f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}
constexpr float kExp2PolyMaxRelErr = 1.123e-04f;
}  // namespace sdpa
