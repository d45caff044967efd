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

}  // namespace ssscan

namespace ssscan {

// ------------------------------------------------------------ mbarrier/TMA ---

// Device error word: a kernel that gives up a bounded wait sets a bit here
// instead of trapping; ss_last_device_error reads and clears it.  (The library
// is a single translation unit, so the definition lives in this header.)
__device__ unsigned int g_error_word = 0;
constexpr unsigned kErrTmaWait = 1u;     // a TMA completion wait timed out
constexpr unsigned kErrLookback = 2u;    // an inter-CTA carry wait timed out
constexpr unsigned kErrBounds = 4u;      // (checked builds) an index outside its tensor

// Checked builds (-DSS_BOUNDS_CHECK): every global index the kernels form is
// compared with its tensor's extent before the access; a miss records
// kErrBounds in the device error word and the access is skipped (no trap, so
// the context stays usable and the host reads the status).  In the product
// build the check is compiled out.
#ifdef SS_BOUNDS_CHECK
__device__ __forceinline__ bool in_range(int64_t i, int64_t n) {
  if (i >= 0 && i < n) return true;
  atomicOr(&g_error_word, kErrBounds);
  return false;
}
#else
__device__ __forceinline__ bool in_range(int64_t, int64_t) { return true; }
#endif
// [i, i + len) inside [0, n)
__device__ __forceinline__ bool in_range(int64_t i, int64_t len, int64_t n) {
  return in_range(i, n) && in_range(i + len - 1, n);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of an mbarrier, giving up after `limit` polls (each
// poll may itself suspend for a hardware-chosen time).  Returns false and
// records kErrTmaWait on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  atomicOr(&g_error_word, kErrTmaWait);
  return false;
}

// One 3-D tiled TMA load (no multicast) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];\n" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// One untiled bulk copy global -> shared (no multicast), completing on `bar`.
// Both addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace ssscan
