// ss_scan.cu -- libssscan.so: the C ABI declared in include/ss_scan.h.  The
// host code of each entry point lives in its *_host.cuh header (forward, decode
// step, backward); this file holds the exported functions and the scratch of
// ss_scan_fwd_noalloc.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "ss_scan.h"
#include "ss_scan_debug.h"
#include "host_common.cuh"
#include "fwd_host.cuh"
#include "step_host.cuh"
#include "bwd_host.cuh"
#include "debug_pointwise.cuh"

using namespace ssscan;

// Scratch of ss_scan_fwd_noalloc: one file-scope device array, held by every
// GPU that loads the library.  Host code must not use its name as an address
// (it is a host-side stand-in); ss_scan_fwd_noalloc looks up the device
// address once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SS_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 128;
std::atomic<void*> g_noalloc_ptr[kMaxDevices];
}  // namespace

extern "C" {

ss_status ss_scan_fwd(const void* u, const void* delta, const float* A, const void* B,
                      const void* C, const float* D, const void* z, const float* delta_bias,
                      int softplus_flag, float* y_out, float* last_state_out, int64_t batch,
                      int64_t dim, int64_t seqlen, int dstate, ss_dtype in_dtype,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return scan_fwd_impl(u, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, y_out,
                       last_state_out, batch, dim, seqlen, dstate, in_dtype, workspace,
                       workspace_bytes, stream);
}

ss_status ss_scan_fwd_from_state(const void* u, const void* delta, const float* A,
                                 const void* B, const void* C, const float* D, const void* z,
                                 const float* delta_bias, int softplus_flag,
                                 const float* initial_state, float* y_out, float* last_state_out,
                                 int64_t batch, int64_t dim, int64_t seqlen, int dstate,
                                 ss_dtype in_dtype, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
  return scan_fwd_impl(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y_out,
                       last_state_out, batch, dim, seqlen, dstate, in_dtype, workspace,
                       workspace_bytes, stream);
}

size_t ss_scan_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen, int dstate) {
  if (batch < 1 || dim < 1 || seqlen < 1 || !supported_dstate(dstate)) return (size_t)-1;
  if (batch > (INT64_C(1) << 40) / dim || batch * dim > (INT64_C(1) << 62) / seqlen)
    return (size_t)-1;
  return ckpt_bytes(batch, dim, seqlen, dstate);
}

ss_status ss_scan_bwd(const void* u, const void* delta, const float* A, const void* B,
                      const void* C, const float* D, const void* z, const float* delta_bias,
                      int softplus_flag, const float* dy, const float* dlast_state,
                      const float* checkpoints, float* du,
                      float* ddelta, float* dA, float* dB, float* dC, float* dD, float* dz,
                      float* ddelta_bias, int64_t batch, int64_t dim, int64_t seqlen, int dstate,
                      ss_dtype in_dtype, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  if (!u || !delta || !A || !B || !C || !dy || !du || !ddelta || !dA || !dB || !dC)
    return SS_ERR_INVALID_ARG;
  if (z && !dz) return SS_ERR_INVALID_ARG;
  if (batch < 1 || dim < 1 || seqlen < 1) return SS_ERR_INVALID_ARG;
  if (in_dtype != SS_F32 && in_dtype != SS_BF16) return SS_ERR_UNSUPPORTED;
  if (!supported_dstate(dstate)) return SS_ERR_UNSUPPORTED;
  if (batch > (INT64_C(1) << 40) / dim || batch * dim > (INT64_C(1) << 62) / seqlen)
    return SS_ERR_INVALID_ARG;
  if (batch * (int64_t)dstate > (INT64_C(1) << 62) / seqlen) return SS_ERR_INVALID_ARG;
  const size_t es = in_dtype == SS_F32 ? 4 : 2;
  const void* in_ptrs[5] = {u, delta, z, B, C};
  for (const void* p : in_ptrs)
    if (p && !aligned(p, es)) return SS_ERR_INVALID_ARG;
  const void* f_ptrs[13] = {A, D, delta_bias, dy, dlast_state, du, ddelta, dA, dB, dC, dD, dz,
                            ddelta_bias};
  for (const void* p : f_ptrs)
    if (p && !aligned(p, 4)) return SS_ERR_INVALID_ARG;
  if (checkpoints ? !aligned(checkpoints, 16) : (!workspace || !aligned(workspace, 256)))
    return SS_ERR_INVALID_ARG;
  // the sums over channels, steps and batch rows accumulate with atomics
  if (cudaMemsetAsync(dA, 0, (size_t)dim * dstate * 4, stream) != cudaSuccess ||
      cudaMemsetAsync(dB, 0, (size_t)(batch * dstate * seqlen) * 4, stream) != cudaSuccess ||
      cudaMemsetAsync(dC, 0, (size_t)(batch * dstate * seqlen) * 4, stream) != cudaSuccess ||
      (dD && cudaMemsetAsync(dD, 0, (size_t)dim * 4, stream) != cudaSuccess) ||
      (ddelta_bias && cudaMemsetAsync(ddelta_bias, 0, (size_t)dim * 4, stream) != cudaSuccess))
    return SS_ERR_CUDA;
  BwdArgs a;
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.A = A; a.D = D; a.delta_bias = delta_bias; a.dy = dy; a.dlast = dlast_state;
  a.du = du; a.ddelta = ddelta; a.dz = dz; a.dA = dA; a.dB = dB; a.dC = dC;
  a.dD = D ? dD : nullptr; a.dbias = ddelta_bias;
  a.ckpt = checkpoints ? const_cast<float*>(checkpoints) : static_cast<float*>(workspace);
  a.ckpt_given = checkpoints != nullptr;
  a.batch = batch; a.dim = dim; a.seqlen = seqlen;
  a.softplus = softplus_flag != 0;
  if (in_dtype == SS_F32) return dispatch_bwd<float>(a, dstate, workspace_bytes, stream);
  return dispatch_bwd<__nv_bfloat16>(a, dstate, workspace_bytes, stream);
}

ss_status ss_scan_fwd_train(const void* u, const void* delta, const float* A, const void* B,
                            const void* C, const float* D, const void* z,
                            const float* delta_bias, int softplus_flag, float* y_out,
                            float* last_state_out, float* checkpoints, int64_t batch, int64_t dim,
                            int64_t seqlen, int dstate, ss_dtype in_dtype, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
  if (!checkpoints || !aligned(checkpoints, 16)) return SS_ERR_INVALID_ARG;
  return scan_fwd_impl(u, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, y_out,
                       last_state_out, batch, dim, seqlen, dstate, in_dtype, workspace,
                       workspace_bytes, stream, nullptr, nullptr, 0, false, checkpoints);
}

ss_status ss_scan_fwd_zoh(const void* u, const void* delta, const float* A, const void* B,
                          const void* C, const float* D, const void* z, const float* delta_bias,
                          int softplus_flag, float* y_out, float* last_state_out, int64_t batch,
                          int64_t dim, int64_t seqlen, int dstate, ss_dtype in_dtype,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return scan_fwd_impl(u, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, y_out,
                       last_state_out, batch, dim, seqlen, dstate, in_dtype, workspace,
                       workspace_bytes, stream, nullptr, nullptr, 0, true);
}

ss_status ss_scan_fwd_conv(const void* x, const float* conv_weight, const float* conv_bias,
                           int conv_width, const void* delta, const float* A, const void* B,
                           const void* C, const float* D, const void* z,
                           const float* delta_bias, int softplus_flag, float* y_out,
                           float* last_state_out, int64_t batch, int64_t dim, int64_t seqlen,
                           int dstate, ss_dtype in_dtype, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
  if (!conv_weight) return SS_ERR_INVALID_ARG;
  return scan_fwd_impl(x, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, y_out,
                       last_state_out, batch, dim, seqlen, dstate, in_dtype, workspace,
                       workspace_bytes, stream, conv_weight, conv_bias, conv_width);
}

ss_status ss_scan_step(const void* u, const void* delta, const float* A, const void* B,
                       const void* C, const float* D, const void* z, const float* delta_bias,
                       int softplus_flag, float* state, float* y_out, int64_t batch, int64_t dim,
                       int dstate, ss_dtype in_dtype, cudaStream_t stream) {
  if (!u || !delta || !A || !B || !C || !state || !y_out) return SS_ERR_INVALID_ARG;
  if (batch < 1 || dim < 1) return SS_ERR_INVALID_ARG;
  if (in_dtype != SS_F32 && in_dtype != SS_BF16) return SS_ERR_UNSUPPORTED;
  if (!supported_dstate(dstate)) return SS_ERR_UNSUPPORTED;
  if (batch > (INT64_C(1) << 56) / dim / dstate) return SS_ERR_INVALID_ARG;
  if (dim * dstate > INT32_MAX) return SS_ERR_INVALID_ARG;  // one row's state indexes in 32 bits
  const size_t es = in_dtype == SS_F32 ? 4 : 2;
  const void* in_ptrs[5] = {u, delta, z, B, C};
  for (const void* p : in_ptrs)
    if (p && !aligned(p, es)) return SS_ERR_INVALID_ARG;
  const void* f_ptrs[5] = {A, D, delta_bias, state, y_out};
  for (const void* p : f_ptrs)
    if (p && !aligned(p, 4)) return SS_ERR_INVALID_ARG;
  StepArgs a;
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.A = A; a.D = D; a.delta_bias = delta_bias;
  a.state = state; a.y = y_out;
  a.batch = batch; a.dim = dim;
  a.softplus = softplus_flag != 0;
  const bool vec = aligned(state, 16) && aligned(A, 16) && aligned(B, 4 * es) && aligned(C, 4 * es);
  // bulk copies need 16-byte aligned sources and sizes: every row of u, delta
  // and z (dim * es bytes) and the state, B, C and A bases
  bool pipe = vec && (dim * (int64_t)es) % 16 == 0 && g_dbg_step_simple.exchange(0) == 0;
  for (const void* p : in_ptrs)
    if (p && !aligned(p, 16)) pipe = false;
  if (in_dtype == SS_F32) return dispatch_step<float>(a, dstate, vec, pipe, stream);
  return dispatch_step<__nv_bfloat16>(a, dstate, vec, pipe, stream);
}

ss_status ss_scan_fwd_noalloc(const void* u, const void* delta, const float* A, const void* B,
                              const void* C, const float* D, const void* z,
                              const float* delta_bias, int softplus_flag, float* y_out,
                              float* last_state_out, int64_t batch, int64_t dim, int64_t seqlen,
                              int dstate, ss_dtype in_dtype, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SS_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SS_ERR_UNSUPPORTED;
  void* scratch = g_noalloc_ptr[dev].load();
  if (!scratch) {  // once per device, with that device current
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch)
      return SS_ERR_CUDA;
    g_noalloc_ptr[dev].store(scratch);
  }
  const size_t need = ss_scan_workspace_bytes(batch, dim, seqlen, dstate);
  if (need != (size_t)-1 && need > SS_NOALLOC_SCRATCH_BYTES) return SS_ERR_UNSUPPORTED;
  // (invalid sizes fall through: ss_scan_fwd rejects them with its own status)
  return ss_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus_flag, y_out, last_state_out,
                     batch, dim, seqlen, dstate, in_dtype, scratch, SS_NOALLOC_SCRATCH_BYTES,
                     stream);
}

size_t ss_scan_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen, int dstate) {
  if (batch < 1 || dim < 1 || seqlen < 1 || !supported_dstate(dstate)) return (size_t)-1;
  if (batch > (INT64_C(1) << 40) / dim || batch * dim > (INT64_C(1) << 62) / seqlen)
    return (size_t)-1;
  // enough for either input dtype and every kernel variant (plain, fused
  // convolution, exact zero-order hold, training checkpoints)
  size_t need[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (!plan_bytes<float, false, false, false>(batch, dim, seqlen, dstate, &need[0]) ||
      !plan_bytes<__nv_bfloat16, false, false, false>(batch, dim, seqlen, dstate, &need[1]) ||
      !plan_bytes<float, true, false, false>(batch, dim, seqlen, dstate, &need[2]) ||
      !plan_bytes<__nv_bfloat16, true, false, false>(batch, dim, seqlen, dstate, &need[3]) ||
      !plan_bytes<float, false, true, false>(batch, dim, seqlen, dstate, &need[4]) ||
      !plan_bytes<__nv_bfloat16, false, true, false>(batch, dim, seqlen, dstate, &need[5]) ||
      !plan_bytes<float, false, false, true>(batch, dim, seqlen, dstate, &need[6]) ||
      !plan_bytes<__nv_bfloat16, false, false, true>(batch, dim, seqlen, dstate, &need[7]))
    return (size_t)-1;
  size_t m = 0;
  for (size_t v : need) m = v > m ? v : m;
  return m;
}

extern "C++" {
namespace {
// The plain forward's plan for this shape (the kernel choice of dispatch_dtype).
template <typename E>
bool fwd_plan(int64_t batch, int64_t dim, int64_t seqlen, int N, ssscan::Plan* p) {
  using namespace ssscan;
  switch (N) {
    case 16:
      return use_time_split<Cfg16<E>>(batch, dim, seqlen) ? make_plan<Split16<E>>(batch, dim, seqlen, p)
                                                          : make_plan<Cfg16<E>>(batch, dim, seqlen, p);
    case 32:
      return use_time_split<Cfg32<E>>(batch, dim, seqlen) ? make_plan<Split32<E>>(batch, dim, seqlen, p)
                                                          : make_plan<Cfg32<E>>(batch, dim, seqlen, p);
    case 64: return make_plan<Cfg64<E>>(batch, dim, seqlen, p);
    case 128: return make_plan<Cfg128<E>>(batch, dim, seqlen, p);
  }
  return false;
}
}  // namespace
}  // extern "C++"

int ss_debug_fwd_kernels(int64_t batch, int64_t dim, int64_t seqlen, int dstate, ss_dtype in_dtype) {
  if (batch < 1 || dim < 1 || seqlen < 1 || !supported_dstate(dstate)) return -1;
  ssscan::Plan p;
  const bool ok = in_dtype == SS_BF16 ? fwd_plan<__nv_bfloat16>(batch, dim, seqlen, dstate, &p)
                                      : fwd_plan<float>(batch, dim, seqlen, dstate, &p);
  if (!ok) return -1;
  return p.nseg > 1 ? 2 : 1;
}

ss_status ss_debug_inject(int what, long long value) {
  switch (what) {
    case SS_DEBUG_FORCE_WORKERS: g_dbg_workers.store(value); return SS_OK;
    case SS_DEBUG_SKIP_PUBLISH: g_dbg_skip_publish.store(value); return SS_OK;
    case SS_DEBUG_SPIN_LIMIT: g_dbg_spin_limit.store(value); return SS_OK;
    case SS_DEBUG_STEP_SIMPLE: g_dbg_step_simple.store(value); return SS_OK;
    case SS_DEBUG_FORCE_SEGMENTS: g_dbg_segments.store(value); return SS_OK;
    case SS_DEBUG_CLEAR:
      g_dbg_segments.store(0);
      g_dbg_step_simple.store(0);
      g_dbg_workers.store(0);
      g_dbg_skip_publish.store(-1);
      g_dbg_spin_limit.store(0);
      return SS_OK;
  }
  return SS_ERR_INVALID_ARG;
}

ss_status ss_debug_pointwise(int fn, const float* x, float* y, int64_t n, cudaStream_t stream) {
  if (fn < kPwSoftplus || fn > kPwEx2 || n < 0 || (n > 0 && (!x || !y))) return SS_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(y, 4)) return SS_ERR_INVALID_ARG;
  if (n == 0) return SS_OK;
  const int64_t pairs = (n + 1) / 2;
  const int64_t blocks = (pairs + 255) / 256 < 4096 ? (pairs + 255) / 256 : 4096;
  pointwise_kernel<<<(unsigned)blocks, 256, 0, stream>>>(fn, x, y, n);
  return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

const char* ss_status_string(ss_status s) {
  switch (s) {
    case SS_OK: return "SS_OK: success";
    case SS_ERR_INVALID_ARG: return "SS_ERR_INVALID_ARG: null pointer, bad size, misalignment or small workspace";
    case SS_ERR_UNSUPPORTED: return "SS_ERR_UNSUPPORTED: dstate must be 16, 32, 64 or 128 and dtype f32 or bf16";
    case SS_ERR_CUDA: return "SS_ERR_CUDA: a CUDA runtime call or launch failed";
    case SS_ERR_TIMEOUT: return "SS_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
    case SS_ERR_BOUNDS: return "SS_ERR_BOUNDS: a checked build met an index outside its tensor";
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
    return (word & kErrBounds) ? SS_ERR_BOUNDS : SS_ERR_TIMEOUT;
  }
  return SS_OK;
}

}  // extern "C"
