// exp2_poly.cuh -- 2^x on the FMA pipe, to relieve the MUFU unit.
// Cody-Waite range reduction (n = round(x) through the 1.5 * 2^23 shifter,
// f = x - n in [-1/2, 1/2]) and a cubic p(f) ~ 2^f with minimax relative
// error, coefficients from fit_exp2_poly.py (Lawson iteration); the result
// is p(f) with n added to its exponent field.  Max relative error 7.48e-05
// for x <= 125; inputs below -125 (-inf included) are clamped to -125,
// giving 2^-125 rather than 0, so masked entries must not come here.
#pragma once
#include <stdint.h>
#include "sm100.cuh"
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
// Two at once: the same steps, each rounded as in exp2_fma, with the
// floating-point ones as packed fp32 pair instructions (identical results).
__device__ __forceinline__ void exp2_fma2(float x0, float x1, float& y0, float& y1) {
  const uint64_t x = f2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t sh = f2_pack(12582912.0f, 12582912.0f);
  const uint64_t t = f2_add(x, sh);
  const uint64_t f = f2_sub(x, f2_sub(t, sh));
  uint64_t p = f2_fma(f2_pack(5.517149344e-02f, 5.517149344e-02f), f,
                      f2_pack(2.426109314e-01f, 2.426109314e-01f));
  p = f2_fma(p, f, f2_pack(6.932609677e-01f, 6.932609677e-01f));
  p = f2_fma(p, f, f2_pack(9.999280572e-01f, 9.999280572e-01f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}
}  // namespace sdpa
