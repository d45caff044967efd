// ss_scan.cu -- host side of libssscan.so: argument checks, kernel choice and
// launch for the C ABI declared in include/ss_scan.h.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cstdint>
#include <cstring>

#include "ss_scan.h"
#include "scan_fwd_chunked.cuh"

namespace ssscan {

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (so the library needs no link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    tried = true;
  }
  return fn;
}

// 3-D map over a [batch][rows][L] tensor, box [1][box_rows][box_t], zero fill
// out of bounds, no swizzle, no multicast.
bool encode_3d(CUtensorMap* m, const void* ptr, bool bf16, int64_t L, int64_t rows,
               int64_t batch, int box_t, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t es = bf16 ? 2 : 4;
  const cuuint64_t dims[3] = {(cuuint64_t)L, (cuuint64_t)rows, (cuuint64_t)batch};
  const cuuint64_t strides[2] = {(cuuint64_t)L * es, (cuuint64_t)L * (cuuint64_t)rows * es};
  const cuuint32_t box[3] = {(cuuint32_t)box_t, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
             const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class CF>
bool encode_maps(const FwdArgs& a, FwdMaps* m) {
  const bool bf16 = sizeof(typename CF::Elem) == 2;
  if (a.seqlen >= INT32_MAX || a.dim >= INT32_MAX || a.batch >= INT32_MAX) return false;
  bool ok = encode_3d(&m->u, a.u, bf16, a.seqlen, a.dim, a.batch, CF::T, CF::CH) &&
            encode_3d(&m->delta, a.delta, bf16, a.seqlen, a.dim, a.batch, CF::T, CF::CH) &&
            encode_3d(&m->z, a.z ? a.z : a.u, bf16, a.seqlen, a.dim, a.batch, CF::T, CF::CH) &&
            encode_3d(&m->B, a.B, bf16, a.seqlen, CF::N, a.batch, CF::T, CF::N) &&
            encode_3d(&m->C, a.C, bf16, a.seqlen, CF::N, a.batch, CF::T, CF::N);
  return ok;
}

template <class CF>
ss_status launch_chunked(FwdArgs a, cudaStream_t stream) {
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
  FwdMaps maps;
  memset(&maps, 0, sizeof maps);
  if (a.vec && !encode_maps<CF>(a, &maps)) a.vec = 0;  // element-wise loads instead
  kern<<<(unsigned)blocks, CF::NT, CF::SMEM_BYTES, stream>>>(a, maps);
  return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

// Launch shapes (lanes per channel K, warps per CTA, chunk length T) per
// state size; the macros exist so that tuning builds can override them.
#ifndef SS_N16_K
#define SS_N16_K 4
#endif
#ifndef SS_N16_W
#define SS_N16_W 4
#endif
#ifndef SS_N16_T
#define SS_N16_T 32
#endif

template <typename E>
ss_status dispatch_dtype(const FwdArgs& a, int N, cudaStream_t stream) {
  // FwdArgs is passed by value so that the launch may switch it to the
  // element-wise path when a tensor map cannot be encoded.
  switch (N) {
    case 16: return launch_chunked<ChunkedCfg<E, 16, SS_N16_K, SS_N16_W, SS_N16_T>>(a, stream);
    case 32: return launch_chunked<ChunkedCfg<E, 32, 4, 4, 32>>(a, stream);
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
