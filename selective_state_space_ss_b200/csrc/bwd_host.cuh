// bwd_host.cuh -- host side of the backward: checkpoint sizes and the launch
// behind ss_scan_bwd
// (host code of libssscan.so; the library is one translation unit, ss_scan.cu)
#pragma once

#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "ss_scan.h"
#include "host_common.cuh"
#include "scan_bwd.cuh"

namespace ssscan {
namespace {

// Checkpoints of the backward: the state at every 16-step chunk start,
// [batch][ceil(L / 16)][dim][N] fp32.
constexpr int kCkptSteps = 16;
size_t ckpt_bytes(int64_t batch, int64_t dim, int64_t seqlen, int N) {
  const int64_t nk = (seqlen + kCkptSteps - 1) / kCkptSteps;
  return align256((size_t)batch * (size_t)nk * (size_t)dim * (size_t)N * sizeof(float));
}

// States per lane of the N = 16 backward (tuning builds may set 2: twice the
// warps; measured faster on B4 L8192 D5120, slower on B8 L2048 D1536 and
// B16 L4096 D2048, so 4 stays the default).
#ifndef SS_BWD_G
#define SS_BWD_G 4
#endif

template <typename E, int N>
ss_status launch_bwd(const BwdArgs& a, size_t ws_bytes, cudaStream_t stream) {
  using CF = BwdCfg<E, N, (N == 16 ? SS_BWD_G : 4)>;
  if (once_per_device<CF>([] {
        return cudaFuncSetAttribute(scan_bwd_kernel<CF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    CF::SMEM_BYTES) == cudaSuccess;
      }) != 1)
    return SS_ERR_CUDA;
  static_assert(CF::T == kCkptSteps, "checkpoint spacing");
  if (!a.ckpt_given && ws_bytes < ckpt_bytes(a.batch, a.dim, a.seqlen, N)) return SS_ERR_INVALID_ARG;
  const int64_t ctas = a.batch * ((a.dim + CF::CH - 1) / CF::CH);
  if (ctas > INT_MAX) return SS_ERR_INVALID_ARG;
  scan_bwd_kernel<CF><<<(unsigned)ctas, CF::NT, CF::SMEM_BYTES, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

template <typename E>
ss_status dispatch_bwd(const BwdArgs& a, int N, size_t ws_bytes, cudaStream_t stream) {
  switch (N) {
    case 16: return launch_bwd<E, 16>(a, ws_bytes, stream);
    case 32: return launch_bwd<E, 32>(a, ws_bytes, stream);
    case 64: return launch_bwd<E, 64>(a, ws_bytes, stream);
    case 128: return launch_bwd<E, 128>(a, ws_bytes, stream);
    default: return SS_ERR_UNSUPPORTED;
  }
}

}  // namespace
}  // namespace ssscan
