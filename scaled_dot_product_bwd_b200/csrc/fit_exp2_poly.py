"""Fit the polynomial of the FMA-pipe exp2 used by the kernels (exp2_poly.cuh).

Method: Cody-Waite range reduction, 2^x = 2^n * 2^f with n = round(x) and
f = x - n in [-1/2, 1/2]; 2^f is approximated by a cubic p(f) whose
coefficients minimise the maximum relative error max |p(f) / 2^f - 1| on
[-1/2, 1/2], found with Lawson's iteratively reweighted least squares (the
weights converge to the minimax solution's).  Prints the coefficients and the
error bound that the GPU test checks; run it to regenerate exp2_poly.cuh.

    python scaled_dot_product_bwd_b200/csrc/fit_exp2_poly.py [--write]
"""
from __future__ import annotations

import os
import sys

import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, iters: int = 400):
    f = np.linspace(-0.5, 0.5, 20001)
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / target[:, None]  # relative error rows
    w = np.ones_like(f) / f.size
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    # coefficients rounded to float32 as the kernel stores them; error of that
    c32 = c.astype(np.float32).astype(np.float64)
    err = np.abs(np.polyval(c32[::-1], f) / target - 1.0).max()
    return c.astype(np.float32), float(err)


HEADER = """// exp2_poly.cuh -- 2^x on the FMA pipe, to relieve the MUFU unit.
// Cody-Waite range reduction (n = round(x) through the 1.5 * 2^23 shifter,
// f = x - n in [-1/2, 1/2]) and a cubic p(f) ~ 2^f with minimax relative
// error, coefficients from fit_exp2_poly.py (Lawson iteration); the result
// is p(f) with n added to its exponent field.  Max relative error {err:.2e}
// for x <= 125; inputs below -125 (-inf included) are clamped to -125,
// giving 2^-125 rather than 0, so masked entries must not come here.
#pragma once
#include <stdint.h>
#include "sm100.cuh"
namespace sdpa {{
__device__ __forceinline__ float exp2_fma(float x) {{
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;  // 1.5 * 2^23: low bits of t hold round(x)
  const float n = t - 12582912.0f;
  const float f = x - n;
  float p = {c3:.9e}f;
  p = fmaf(p, f, {c2:.9e}f);
  p = fmaf(p, f, {c1:.9e}f);
  p = fmaf(p, f, {c0:.9e}f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}}
constexpr float kExp2PolyMaxRelErr = {bound:.3e}f;
// Two at once: the same steps, each rounded as in exp2_fma, with the
// floating-point ones as packed fp32 pair instructions (identical results).
__device__ __forceinline__ void exp2_fma2(float x0, float x1, float& y0, float& y1) {{
  const uint64_t x = f2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t sh = f2_pack(12582912.0f, 12582912.0f);
  const uint64_t t = f2_add(x, sh);
  const uint64_t f = f2_sub(x, f2_sub(t, sh));
  uint64_t p = f2_fma(f2_pack({c3:.9e}f, {c3:.9e}f), f,
                      f2_pack({c2:.9e}f, {c2:.9e}f));
  p = f2_fma(p, f, f2_pack({c1:.9e}f, {c1:.9e}f));
  p = f2_fma(p, f, f2_pack({c0:.9e}f, {c0:.9e}f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}}
}}  // namespace sdpa
"""


def main():
    c, err = fit()
    print("coefficients c0..c3:", [float(x) for x in c])
    print(f"max relative error on [-1/2, 1/2]: {err:.3e}")
    if "--write" in sys.argv:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "exp2_poly.cuh")
        with open(path, "w") as fh:
            fh.write(HEADER.format(err=err, c0=c[0], c1=c[1], c2=c[2], c3=c[3], bound=err * 1.5))
        print("wrote", path)


if __name__ == "__main__":
    main()
