// ss_scan.cu -- host side of libssscan.so: argument checks, kernel choice and
// launch for the C ABI declared in include/ss_scan.h.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>
#include <cstring>

#include "ss_scan.h"
#include "scan_fwd_chunked.cuh"

namespace ssscan {

// Device error word: a kernel that gives up a bounded wait ORs in a code;
// ss_last_device_error reads and clears it.
__device__ unsigned int g_error_word = 0;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <class CF>
ss_status launch_chunked(const FwdArgs& a, cudaStream_t stream) {
  static bool configured = false;  // one attribute call per instantiation and process
  auto kern = scan_fwd_chunked_kernel<CF>;
  if (!configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, CF::SMEM_BYTES) !=
        cudaSuccess)
      return SS_ERR_CUDA;
    configured = true;
  }
  const int64_t tiles = (a.dim + CF::CH - 1) / CF::CH;
  const int64_t blocks = tiles * a.batch;
  if (blocks > INT_MAX) return SS_ERR_INVALID_ARG;
  kern<<<(unsigned)blocks, CF::NT, CF::SMEM_BYTES, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

template <typename E>
ss_status dispatch_dtype(const FwdArgs& a, int N, cudaStream_t stream) {
  switch (N) {
    case 16: return launch_chunked<ChunkedCfg<E, 16, 4, 4, 64>>(a, stream);
    case 32: return launch_chunked<ChunkedCfg<E, 32, 4, 4, 64>>(a, stream);
    case 64: return launch_chunked<ChunkedCfg<E, 64, 8, 8, 32>>(a, stream);
    case 128: return launch_chunked<ChunkedCfg<E, 128, 8, 8, 32>>(a, stream);
    default: return SS_ERR_UNSUPPORTED;
  }
}

bool supported_dstate(int n) { return n == 16 || n == 32 || n == 64 || n == 128; }

}  // namespace
}  // namespace ssscan

using namespace ssscan;

extern "C" {

ss_status ss_scan_fwd(const void* u, const void* delta, const float* A, const void* B,
                      const void* C, const float* D, const void* z, const float* delta_bias,
                      int softplus_flag, float* y_out, float* last_state_out, int64_t batch,
                      int64_t dim, int64_t seqlen, int dstate, ss_dtype in_dtype,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!u || !delta || !A || !B || !C || !y_out) return SS_ERR_INVALID_ARG;
  if (batch < 1 || dim < 1 || seqlen < 1) return SS_ERR_INVALID_ARG;
  if (in_dtype != SS_F32 && in_dtype != SS_BF16) return SS_ERR_UNSUPPORTED;
  if (!supported_dstate(dstate)) return SS_ERR_UNSUPPORTED;
  // batch*dim*seqlen and batch*dstate*seqlen must stay far from int64 overflow
  if (batch > (INT64_C(1) << 40) / dim || batch * dim > (INT64_C(1) << 62) / seqlen)
    return SS_ERR_INVALID_ARG;
  if (batch * (int64_t)dstate > (INT64_C(1) << 62) / seqlen) return SS_ERR_INVALID_ARG;
  const size_t es = in_dtype == SS_F32 ? 4 : 2;
  const void* in_ptrs[5] = {u, delta, z, B, C};
  for (const void* p : in_ptrs)
    if (p && !aligned(p, es)) return SS_ERR_INVALID_ARG;
  const void* f_ptrs[5] = {A, D, delta_bias, y_out, last_state_out};
  for (const void* p : f_ptrs)
    if (p && !aligned(p, 4)) return SS_ERR_INVALID_ARG;
  const size_t need = ss_scan_workspace_bytes(batch, dim, seqlen, dstate);
  if (need == (size_t)-1) return SS_ERR_INVALID_ARG;
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
    return SS_ERR_INVALID_ARG;

  FwdArgs a;
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.A = A; a.D = D; a.delta_bias = delta_bias;
  a.y = y_out; a.last_state = last_state_out;
  a.batch = batch; a.dim = dim; a.seqlen = seqlen;
  a.softplus = softplus_flag != 0;
  bool vec = ((size_t)seqlen * es) % 16 == 0;
  for (const void* p : in_ptrs)
    if (p && !aligned(p, 16)) vec = false;
  if (!aligned(y_out, 16)) vec = false;
  a.vec = vec ? 1 : 0;

  if (in_dtype == SS_F32) return dispatch_dtype<float>(a, dstate, stream);
  return dispatch_dtype<__nv_bfloat16>(a, dstate, stream);
}

size_t ss_scan_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen, int dstate) {
  if (batch < 1 || dim < 1 || seqlen < 1 || !supported_dstate(dstate)) return (size_t)-1;
  return 0;
}

const char* ss_status_string(ss_status s) {
  switch (s) {
    case SS_OK: return "SS_OK: success";
    case SS_ERR_INVALID_ARG: return "SS_ERR_INVALID_ARG: null pointer, bad size, misalignment or small workspace";
    case SS_ERR_UNSUPPORTED: return "SS_ERR_UNSUPPORTED: dstate must be 16, 32, 64 or 128 and dtype f32 or bf16";
    case SS_ERR_CUDA: return "SS_ERR_CUDA: a CUDA runtime call or launch failed";
    case SS_ERR_TIMEOUT: return "SS_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
  }
  return "unknown ss_status";
}

ss_status ss_last_device_error(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SS_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof word) != cudaSuccess) return SS_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof zero) != cudaSuccess) return SS_ERR_CUDA;
    return SS_ERR_TIMEOUT;
  }
  return SS_OK;
}

}  // extern "C"
