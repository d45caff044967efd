// debug_pointwise.cuh -- element-wise evaluation of the kernels' pointwise
// functions (pointwise.cuh), so that tests can check each approximation
// against float64 over its whole input range.  Not used by any scan.
#pragma once

#include "pointwise.cuh"

namespace ssscan {

// Which function ss_debug_pointwise evaluates (include/ss_scan_debug.h).
enum : int {
  kPwSoftplus = 0,      // softplus_fast
  kPwSilu = 1,          // silu_fast
  kPwSoftplus2 = 2,     // softplus_fast2 on pairs (x[2i], x[2i+1])
  kPwSilu2 = 3,         // silu_fast2 on pairs
  kPwExp2NegFma = 4,    // exp2_neg_fma2 on pairs (2^x for x <= 0 on the FMA pipe)
  kPwRcp12 = 5,         // rcp_1_2 (1/d for d in [1, 2], Newton-Raphson)
  kPwEx2 = 6,           // ex2.approx (the special-function unit's 2^x)
};

__global__ void pointwise_kernel(int fn, const float* __restrict__ x, float* __restrict__ y,
                                 int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; 2 * i < n; i += stride) {
    const int64_t i0 = 2 * i, i1 = 2 * i + 1;
    const float a = x[i0], b = i1 < n ? x[i1] : 0.f;
    float2 r;
    switch (fn) {
      case kPwSoftplus: r = make_float2(softplus_fast(a), softplus_fast(b)); break;
      case kPwSilu: r = make_float2(silu_fast(a), silu_fast(b)); break;
      case kPwSoftplus2: r = softplus_fast2(make_float2(a, b)); break;
      case kPwSilu2: r = silu_fast2(make_float2(a, b)); break;
      case kPwExp2NegFma: r = exp2_neg_fma2(make_float2(a, b)); break;
      case kPwRcp12: r = make_float2(rcp_1_2(a), rcp_1_2(b)); break;
      default: r = make_float2(ex2_approx(a), ex2_approx(b)); break;
    }
    y[i0] = r.x;
    if (i1 < n) y[i1] = r.y;
  }
}

}  // namespace ssscan
