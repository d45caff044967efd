// scan_common.cuh -- small device helpers shared by the selective-scan kernels.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace ssscan {

constexpr unsigned kFullMask = 0xffffffffu;

// 2^x on the special-function unit (approximate, flushes subnormals to 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 16-byte asynchronous global->shared copy (L2 only, no L1 allocation).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Four consecutive stored elements from shared memory, widened to float.
__device__ __forceinline__ float4 load4_f32(const float* s) { return *reinterpret_cast<const float4*>(s); }
__device__ __forceinline__ float4 load4_f32(const __nv_bfloat16* s) {
  const uint2 v = *reinterpret_cast<const uint2*>(s);
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                     __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T zero_elem();
template <> __device__ __forceinline__ float zero_elem<float>() { return 0.f; }
template <> __device__ __forceinline__ __nv_bfloat16 zero_elem<__nv_bfloat16>() { return __float2bfloat16_rn(0.f); }

// softplus(x) = log(1 + e^x); above 20 the correction e^-x is below half an
// fp32 ulp of x, so x itself is returned.
__device__ __forceinline__ float softplus_f32(float x) { return x > 20.f ? x : log1pf(expf(x)); }

// SiLU(z) = z * sigmoid(z) = z / (1 + e^-z).
__device__ __forceinline__ float silu_f32(float z) { return z / (1.f + expf(-z)); }

}  // namespace ssscan
