// pointwise.cuh -- per-element math of the scan epilogue/prologue with one
// special-function-unit (MUFU) operation each.  The scan is bound by the MUFU
// rate (one ex2 per state and step), so the rest of the pointwise math runs on
// the FMA pipe: the log1p of softplus as a polynomial, the reciprocal of the
// sigmoid by Newton-Raphson.  Constants come from csrc/fit_poly.py.
#pragma once

#include "scan_common.cuh"

namespace ssscan {

// log1p(e)/e on e in [0,1], degree 8, float32 Horner: max rel err 1.7e-7.
__device__ __forceinline__ float log1p_unit(float e) {
  float p = 5.105825607e-03f;
  p = fmaf(p, e, -2.899195626e-02f);
  p = fmaf(p, e, 7.738073915e-02f);
  p = fmaf(p, e, -1.359059960e-01f);
  p = fmaf(p, e, 1.907130927e-01f);
  p = fmaf(p, e, -2.483394593e-01f);
  p = fmaf(p, e, 3.331793547e-01f);
  p = fmaf(p, e, -4.999943674e-01f);
  p = fmaf(p, e, 9.999999404e-01f);
  return p * e;
}

// softplus(x) = log(1 + e^x) = max(x, 0) + log1p(e^-|x|).  The ex2 argument
// is -|x| log2(e) <= 0; below -126 the flush-to-zero ex2 returns 0 and the
// result is max(x, 0), exact to fp32.
__device__ __forceinline__ float softplus_fast(float x) {
  const float e = ex2_approx(-fabsf(x) * 1.4426950408889634f);
  return fmaxf(x, 0.f) + log1p_unit(e);
}

// 1/d for d in [1, 2]: linear seed 24/17 - 8/17 d (the minimax line for the
// reciprocal, relative error <= 1/17), then three Newton-Raphson steps
// r <- r + r (1 - d r); the error squares each step: 1/17 -> 3.5e-3 ->
// 1.2e-5 -> 1.5e-10, below fp32 rounding.
__device__ __forceinline__ float rcp_1_2(float d) {
  float r = fmaf(-0.4705882352941176f, d, 1.4117647058823530f);
  float t = fmaf(-d, r, 1.f);
  r = fmaf(r, t, r);
  t = fmaf(-d, r, 1.f);
  r = fmaf(r, t, r);
  t = fmaf(-d, r, 1.f);
  r = fmaf(r, t, r);
  return r;
}

// SiLU(z) = z sigmoid(z); with e = e^-|z| in (0, 1]:
// sigmoid(z) = 1/(1+e) for z >= 0 and e/(1+e) for z < 0.  The reciprocal of
// 1+e in (1, 2] is taken on the special-function unit (one instruction,
// ~1 ulp); rcp_1_2 is the FMA-pipe alternative for kernels bound by that unit.
__device__ __forceinline__ float silu_fast(float z) {
  const float e = ex2_approx(-fabsf(z) * 1.4426950408889634f);
  const float r = rcp_approx(1.f + e);
  return z * (z >= 0.f ? r : e * r);
}

}  // namespace ssscan
