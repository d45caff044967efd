// step_host.cuh -- host side of the recurrent decode step: kernel choice and
// launch behind ss_scan_step
// (host code of libssscan.so; the library is one translation unit, ss_scan.cu)
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdint>

#include "ss_scan.h"
#include "host_common.cuh"
#include "scan_step.cuh"

namespace ssscan {
namespace {

template <typename E, int N>
ss_status launch_step(const StepArgs& a, bool vec, cudaStream_t stream) {
  constexpr int64_t per_block = kStepThreads * kStepUnits;
  const int64_t bx = (a.dim * (N / 4) + per_block - 1) / per_block;
  if (bx > INT_MAX) return SS_ERR_INVALID_ARG;
  const dim3 grid((unsigned)bx, (unsigned)(a.batch < 65535 ? a.batch : 65535));
  if (vec) scan_step_kernel<E, N, true><<<grid, kStepThreads, 0, stream>>>(a);
  else scan_step_kernel<E, N, false><<<grid, kStepThreads, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

// The bulk-copy pipeline: persistent CTAs, as many as fit on the device at once.
template <typename E, int N>
ss_status launch_step_pipe(const StepArgs& a, cudaStream_t stream) {
  using CF = StepPipeCfg<E, N>;
  if (once_per_device<CF>([] {
        return cudaFuncSetAttribute(scan_step_pipe_kernel<E, N>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    CF::SMEM_BYTES) == cudaSuccess;
      }) != 1)
    return SS_ERR_CUDA;
  static std::atomic<int> occ_cache[kDevCache];  // resident CTAs per SM, per device
  int dev = 0, occ = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SS_ERR_CUDA;
  if (dev >= 0 && dev < kDevCache) occ = occ_cache[dev].load();
  if (occ < 1) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, scan_step_pipe_kernel<E, N>,
                                                      CF::THREADS, CF::SMEM_BYTES) != cudaSuccess ||
        occ < 1)
      return SS_ERR_CUDA;
    if (dev >= 0 && dev < kDevCache) occ_cache[dev].store(occ);
  }
  StepPipeSched sc;
  sc.tiles_per_row = (a.dim + CF::TILE_CH - 1) / CF::TILE_CH;
  sc.items = sc.tiles_per_row * a.batch;
  const int64_t slots = (int64_t)device_sms() * occ;
  if (slots < 1) return SS_ERR_CUDA;
  const int64_t grid = sc.items < slots ? sc.items : slots;
  // a programmatic dependent launch: the grid may start while the previous
  // kernel in the stream drains; the kernel waits for it before any read
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(CF::THREADS);
  cfg.dynamicSmemBytes = CF::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, scan_step_pipe_kernel<E, N>, a, sc) != cudaSuccess) return SS_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

template <typename E>
ss_status dispatch_step(const StepArgs& a, int N, bool vec, bool pipe, cudaStream_t stream) {
  switch (N) {
    case 16: return pipe ? launch_step_pipe<E, 16>(a, stream) : launch_step<E, 16>(a, vec, stream);
    case 32: return pipe ? launch_step_pipe<E, 32>(a, stream) : launch_step<E, 32>(a, vec, stream);
    case 64: return pipe ? launch_step_pipe<E, 64>(a, stream) : launch_step<E, 64>(a, vec, stream);
    case 128: return pipe ? launch_step_pipe<E, 128>(a, stream) : launch_step<E, 128>(a, vec, stream);
    default: return SS_ERR_UNSUPPORTED;
  }
}

}  // namespace
}  // namespace ssscan
