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

// 2^x for x <= 0 on the FMA pipe (no special-function unit): x is clamped
// to -126 (2^-126 ~ 1.2e-38 stands for 0 here), split as x = k + f with
// k = round(x) by the 1.5 * 2^23 magic-number rounding and f in [-0.5, 0.5];
// 2^f is the degree-6 fit of csrc/fit_poly.py (max rel err 9.7e-8) and 2^k is
// put straight into the exponent field.
__device__ __forceinline__ float2 exp2_neg_fma2(float2 x) {
  x = make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f));
  const float2 magic = make_float2(12582912.f, 12582912.f);
  const float2 j = __fadd2_rn(x, magic);
  const float2 k = __fadd2_rn(j, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(k, make_float2(-1.f, -1.f), x);
  float2 p = make_float2(1.533757750e-04f, 1.533757750e-04f);
  p = __ffma2_rn(p, f, make_float2(1.339985989e-03f, 1.339985989e-03f));
  p = __ffma2_rn(p, f, make_float2(9.618519805e-03f, 9.618519805e-03f));
  p = __ffma2_rn(p, f, make_float2(5.550329015e-02f, 5.550329015e-02f));
  p = __ffma2_rn(p, f, make_float2(2.402264625e-01f, 2.402264625e-01f));
  p = __ffma2_rn(p, f, make_float2(6.931471825e-01f, 6.931471825e-01f));
  p = __ffma2_rn(p, f, make_float2(1.f, 1.f));
  // bits of j are 0x4B400000 + k; (k + 127) << 23 is the exponent of 2^k
  const int kx = __float_as_int(j.x) - 0x4B400000 + 127;
  const int ky = __float_as_int(j.y) - 0x4B400000 + 127;
  return __fmul2_rn(p, make_float2(__int_as_float(kx << 23), __int_as_float(ky << 23)));
}

// ---- packed forms: two independent elements per fp32x2 operation ----

__device__ __forceinline__ float2 fabs2(float2 v) { return make_float2(fabsf(v.x), fabsf(v.y)); }

// log1p(e)/e polynomial (same constants as log1p_unit) on a pair.
__device__ __forceinline__ float2 log1p_unit2(float2 e) {
  float2 p = make_float2(5.105825607e-03f, 5.105825607e-03f);
  p = __ffma2_rn(p, e, make_float2(-2.899195626e-02f, -2.899195626e-02f));
  p = __ffma2_rn(p, e, make_float2(7.738073915e-02f, 7.738073915e-02f));
  p = __ffma2_rn(p, e, make_float2(-1.359059960e-01f, -1.359059960e-01f));
  p = __ffma2_rn(p, e, make_float2(1.907130927e-01f, 1.907130927e-01f));
  p = __ffma2_rn(p, e, make_float2(-2.483394593e-01f, -2.483394593e-01f));
  p = __ffma2_rn(p, e, make_float2(3.331793547e-01f, 3.331793547e-01f));
  p = __ffma2_rn(p, e, make_float2(-4.999943674e-01f, -4.999943674e-01f));
  p = __ffma2_rn(p, e, make_float2(9.999999404e-01f, 9.999999404e-01f));
  return __fmul2_rn(p, e);
}

#ifndef SS_POINTWISE_MUFU
#define SS_POINTWISE_MUFU 3  // special-function ops per element in softplus + SiLU
#endif

// softplus on a pair (same math as softplus_fast).
__device__ __forceinline__ float2 softplus_fast2(float2 x) {
  const float2 t = __fmul2_rn(fabs2(x), make_float2(-1.4426950408889634f, -1.4426950408889634f));
#if SS_POINTWISE_MUFU >= 3
  const float2 e = make_float2(ex2_approx(t.x), ex2_approx(t.y));
#else
  const float2 e = exp2_neg_fma2(t);
#endif
  return __fadd2_rn(make_float2(fmaxf(x.x, 0.f), fmaxf(x.y, 0.f)), log1p_unit2(e));
}

// SiLU on a pair (same math as silu_fast).
__device__ __forceinline__ float2 silu_fast2(float2 z) {
  const float2 t = __fmul2_rn(fabs2(z), make_float2(-1.4426950408889634f, -1.4426950408889634f));
#if SS_POINTWISE_MUFU >= 2
  const float2 e = make_float2(ex2_approx(t.x), ex2_approx(t.y));
#else
  const float2 e = exp2_neg_fma2(t);
#endif
  const float2 d = __fadd2_rn(e, make_float2(1.f, 1.f));
#if SS_POINTWISE_MUFU >= 3
  const float2 r = make_float2(rcp_approx(d.x), rcp_approx(d.y));
#else
  const float2 r = make_float2(rcp_1_2(d.x), rcp_1_2(d.y));
#endif
  const float2 er = __fmul2_rn(e, r);
  const float2 sg = make_float2(z.x >= 0.f ? r.x : er.x, z.y >= 0.f ? r.y : er.y);
  return __fmul2_rn(z, sg);
}

}  // namespace ssscan
