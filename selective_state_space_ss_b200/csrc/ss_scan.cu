// ss_scan.cu -- host side of libssscan.so: argument checks, kernel choice and
// launch for the C ABI declared in include/ss_scan.h.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <chrono>
#include <climits>
#include <cstdint>
#include <cstring>

#include "ss_scan.h"
#include "ss_scan_debug.h"
#include "scan_fwd_chunked.cuh"
#include "scan_step.cuh"
#include "scan_bwd.cuh"

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
  bool ok = encode_3d(&m->u, a.u, bf16, a.seqlen, a.dim, a.batch, CF::XT, CF::CH) &&
            encode_3d(&m->delta, a.delta, bf16, a.seqlen, a.dim, a.batch, CF::T, CF::CH) &&
            encode_3d(&m->z, a.z ? a.z : a.u, bf16, a.seqlen, a.dim, a.batch, CF::T, CF::CH) &&
            encode_3d(&m->B, a.B, bf16, a.seqlen, CF::N, a.batch, CF::T, CF::N) &&
            encode_3d(&m->C, a.C, bf16, a.seqlen, CF::N, a.batch, CF::T, CF::N);
  return ok;
}

// Test hooks (ss_scan_debug.h): consumed by the next ss_scan_fwd call.
std::atomic<long long> g_dbg_workers{0};
std::atomic<long long> g_dbg_skip_publish{-1};
std::atomic<long long> g_dbg_spin_limit{0};
std::atomic<long long> g_dbg_step_simple{0};

constexpr uint32_t kCarrySpinLimit = 1u << 22;  // ~1 s of polling with back-off

// A launch-unique 64-bit epoch: carry flags written by earlier launches (or
// arbitrary bytes in a fresh workspace) never equal it.
unsigned long long next_epoch() {
  static std::atomic<unsigned long long> ctr{
      (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() *
      0x9E3779B97F4A7C15ULL};
  return ctr.fetch_add(0x9E3779B97F4A7C15ULL) | 1ULL;
}

// Per-device answers that never change, looked up once (every launch plans its
// schedule, and every workspace query plans all kernel variants).
constexpr int kDevCache = 64;

int device_sms() {
  static std::atomic<int> cache[kDevCache];
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kDevCache && (sms = cache[dev].load()) > 0) return sms;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kDevCache) cache[dev].store(sms);
  return sms;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Run `setup` (attribute settings of a kernel family) once per device: the
// dynamic shared memory limit is a per-device setting, so a process that
// drives several GPUs needs it on each.  `Tag` keeps one cache per family.
// Returns the cached value: 1 set up, -1 failed.
template <class Tag, class F>
int once_per_device(F setup) {
  static std::atomic<int> state[kDevCache];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev < 0 || dev >= kDevCache) return setup() ? 1 : -1;  // not cached
  int v = state[dev].load();
  if (v == 0) {
    v = setup() ? 1 : -1;  // idempotent: a concurrent first call may repeat it
    state[dev].store(v);
  }
  return v;
}

// How the work is cut: `workers` CTAs, each an equal contiguous range of
// (channel group, chunk) units.  workers == groups means one group per CTA and
// no carries; fewer workers balance the load across SMs with carry handoff.
struct Plan {
  int workers = 0;
  int64_t groups = 0, nk = 0, tiles = 0;
  size_t carry_bytes = 0, ws_bytes = 0;
};

template <class CF>
bool configure_kernel() {
  return once_per_device<CF>([] {
    return cudaFuncSetAttribute(scan_fwd_chunked_kernel<CF, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                CF::SMEM_BYTES) == cudaSuccess &&
           cudaFuncSetAttribute(scan_fwd_chunked_kernel<CF, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                CF::SMEM_BYTES) == cudaSuccess;
  }) == 1;
}

template <class CF>
bool make_plan(int64_t batch, int64_t dim, int64_t seqlen, Plan* p) {
  if (!configure_kernel<CF>()) return false;
  p->tiles = (dim + CF::CH - 1) / CF::CH;
  p->groups = batch * p->tiles;
  p->nk = (seqlen + CF::T - 1) / CF::T;
  static std::atomic<int> occ_cache[kDevCache];  // resident CTAs per SM, per device
  int dev = 0, occ = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < kDevCache) occ = occ_cache[dev].load();
  if (occ < 1) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, scan_fwd_chunked_kernel<CF, true>, CF::NT,
                                                      CF::SMEM_BYTES) != cudaSuccess || occ < 1)
      return false;
    if (dev >= 0 && dev < kDevCache) occ_cache[dev].store(occ);
  }
  const int64_t sms = device_sms();
  if (sms < 1) return false;
  // One group per CTA (the plain loop) unless the work is between one and two
  // waves of CTAs with the second at most half full: then one persistent CTA
  // per resident slot, with balanced ranges and carry handoff, instead of a
  // nearly empty extra round.  (Measured: the balanced loop costs ~7 % per
  // chunk in bookkeeping; at 2-3 CTAs per SM fewer, balanced workers lose more
  // in occupancy than the tail costs; over several waves the block scheduler
  // already spreads the tail.)
  const int64_t slots = sms * occ;
  int64_t w = p->groups;
  if (p->groups > slots && p->groups < 2 * slots && 2 * (p->groups - slots) <= slots) w = slots;
  const long long forced = g_dbg_workers.load();
  if (forced > 0) w = forced < p->groups ? forced : p->groups;
  if (w > INT_MAX || p->groups > INT32_MAX || p->nk > INT32_MAX) return false;
  p->workers = (int)w;
  if (p->workers < p->groups) {
    p->carry_bytes = align256((size_t)p->workers * CF::CH * CF::N * sizeof(float));
    p->ws_bytes = p->carry_bytes + align256((size_t)p->workers * sizeof(unsigned long long));
  }
  return true;
}

template <class CF>
ss_status launch_chunked(FwdArgs a, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
  Plan p;
  if (!make_plan<CF>(a.batch, a.dim, a.seqlen, &p)) return SS_ERR_CUDA;
  if (p.ws_bytes > 0 && (!workspace || workspace_bytes < p.ws_bytes ||
                         !aligned(workspace, 256)))
    return SS_ERR_INVALID_ARG;
  FwdMaps maps;
  memset(&maps, 0, sizeof maps);
  if (a.vec && !encode_maps<CF>(a, &maps)) a.vec = 0;  // element-wise loads instead
  Sched sc;
  sc.units = p.groups * p.nk;
  sc.nk = p.nk;
  sc.tiles_per_b = p.tiles;
  sc.carries = p.ws_bytes ? static_cast<float*>(workspace) : nullptr;
  sc.flags = p.ws_bytes ? reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) +
                                                                 p.carry_bytes)
                        : nullptr;
  sc.epoch = next_epoch();
  const long long spin = g_dbg_spin_limit.exchange(0);
  sc.spin_limit = spin > 0 ? (uint32_t)spin : kCarrySpinLimit;
  sc.skip_publish = (int)g_dbg_skip_publish.exchange(-1);
  g_dbg_workers.store(0);
  if (p.workers == p.groups)
    scan_fwd_chunked_kernel<CF, false><<<(unsigned)p.workers, CF::NT, CF::SMEM_BYTES, stream>>>(a, maps, sc);
  else
    scan_fwd_chunked_kernel<CF, true><<<(unsigned)p.workers, CF::NT, CF::SMEM_BYTES, stream>>>(a, maps, sc);
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

template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Cfg16 = ChunkedCfg<E, 16, SS_N16_K, SS_N16_W, SS_N16_T, 1, CV, Z, TR>;
#ifndef SS_N32_K
#define SS_N32_K 4
#endif
#ifndef SS_N32_W
#define SS_N32_W 4
#endif
#ifndef SS_N32_T
#define SS_N32_T 32
#endif
template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Cfg32 = ChunkedCfg<E, 32, SS_N32_K, SS_N32_W, SS_N32_T, 1, CV, Z, TR>;
#ifndef SS_N64_K
#define SS_N64_K 4
#endif
#ifndef SS_N64_W
#define SS_N64_W 4
#endif
#ifndef SS_N64_T
#define SS_N64_T 32
#endif
#ifndef SS_N128_K
#define SS_N128_K 16
#endif
#ifndef SS_N128_W
#define SS_N128_W 8
#endif
#ifndef SS_N128_T
#define SS_N128_T 32
#endif
template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Cfg64 = ChunkedCfg<E, 64, SS_N64_K, SS_N64_W, SS_N64_T, 1, CV, Z, TR>;
template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Cfg128 = ChunkedCfg<E, 128, SS_N128_K, SS_N128_W, SS_N128_T, 1, CV, Z, TR>;

// Time-split shapes for problems with too few channels to fill the GPU: one
// warp's worth of channels (8) per CTA, 8 warps splitting each chunk in time.
#ifndef SS_SPLIT16_W
#define SS_SPLIT16_W 8
#endif
#ifndef SS_SPLIT16_T
#define SS_SPLIT16_T 128
#endif
#ifndef SS_SPLIT16_WT
#define SS_SPLIT16_WT 8
#endif
template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Split16 = ChunkedCfg<E, 16, 4, SS_SPLIT16_W, SS_SPLIT16_T, SS_SPLIT16_WT, CV, Z, TR>;
template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Split32 = ChunkedCfg<E, 32, 4, 8, 32, 8, CV, Z, TR>;

// The time split costs ~1.5 extra instructions per (step, state); take it only
// when the channel-parallel shape would leave SMs idle.
template <class CF>
bool too_few_groups(int64_t batch, int64_t dim) {
#ifdef SS_SPLIT_ALWAYS
  return true;
#endif
  const int64_t groups = batch * ((dim + CF::CH - 1) / CF::CH);
  return groups < device_sms();
}

template <typename E, bool CV, bool Z, bool TR>
ss_status dispatch_dtype(const FwdArgs& a, int N, void* ws, size_t wsb, cudaStream_t stream) {
  switch (N) {
    case 16:
      if (too_few_groups<Cfg16<E, CV, Z, TR>>(a.batch, a.dim))
        return launch_chunked<Split16<E, CV, Z, TR>>(a, ws, wsb, stream);
      return launch_chunked<Cfg16<E, CV, Z, TR>>(a, ws, wsb, stream);
    case 32:
      if (too_few_groups<Cfg32<E, CV, Z, TR>>(a.batch, a.dim))
        return launch_chunked<Split32<E, CV, Z, TR>>(a, ws, wsb, stream);
      return launch_chunked<Cfg32<E, CV, Z, TR>>(a, ws, wsb, stream);
    case 64: return launch_chunked<Cfg64<E, CV, Z, TR>>(a, ws, wsb, stream);
    case 128: return launch_chunked<Cfg128<E, CV, Z, TR>>(a, ws, wsb, stream);
    default: return SS_ERR_UNSUPPORTED;
  }
}

template <typename E, bool CV, bool Z, bool TR>
bool plan_bytes(int64_t batch, int64_t dim, int64_t seqlen, int N, size_t* bytes) {
  Plan p;
  bool ok = false;
  switch (N) {
    case 16:
      ok = too_few_groups<Cfg16<E, CV, Z, TR>>(batch, dim) ? make_plan<Split16<E, CV, Z, TR>>(batch, dim, seqlen, &p)
                                                    : make_plan<Cfg16<E, CV, Z, TR>>(batch, dim, seqlen, &p);
      break;
    case 32:
      ok = too_few_groups<Cfg32<E, CV, Z, TR>>(batch, dim) ? make_plan<Split32<E, CV, Z, TR>>(batch, dim, seqlen, &p)
                                                    : make_plan<Cfg32<E, CV, Z, TR>>(batch, dim, seqlen, &p);
      break;
    case 64: ok = make_plan<Cfg64<E, CV, Z, TR>>(batch, dim, seqlen, &p); break;
    case 128: ok = make_plan<Cfg128<E, CV, Z, TR>>(batch, dim, seqlen, &p); break;
  }
  *bytes = p.ws_bytes;
  return ok;
}

bool supported_dstate(int n) { return n == 16 || n == 32 || n == 64 || n == 128; }

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
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, scan_step_pipe_kernel<E, N>, CF::NT,
                                                      CF::SMEM_BYTES) != cudaSuccess || occ < 1)
      return SS_ERR_CUDA;
    if (dev >= 0 && dev < kDevCache) occ_cache[dev].store(occ);
  }
  StepPipeSched sc;
  sc.tiles_per_row = (a.dim + CF::TILE_CH - 1) / CF::TILE_CH;
  sc.items = sc.tiles_per_row * a.batch;
  const int64_t slots = (int64_t)device_sms() * occ;
  if (slots < 1) return SS_ERR_CUDA;
  const int64_t grid = sc.items < slots ? sc.items : slots;
  scan_step_pipe_kernel<E, N><<<(unsigned)grid, CF::NT, CF::SMEM_BYTES, stream>>>(a, sc);
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

// Checkpoints of the backward: the state at every 16-step chunk start,
// [batch][ceil(L / 16)][dim][N] fp32.
constexpr int kCkptSteps = 16;
size_t ckpt_bytes(int64_t batch, int64_t dim, int64_t seqlen, int N) {
  const int64_t nk = (seqlen + kCkptSteps - 1) / kCkptSteps;
  return align256((size_t)batch * (size_t)nk * (size_t)dim * (size_t)N * sizeof(float));
}

template <typename E, int N>
ss_status launch_bwd(const BwdArgs& a, size_t ws_bytes, cudaStream_t stream) {
  using CF = BwdCfg<E, N>;
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

ss_status scan_fwd_impl(const void* u, const void* delta, const float* A, const void* B,
                        const void* C, const float* D, const void* z, const float* delta_bias,
                        int softplus_flag, const float* h0, float* y_out, float* last_state_out,
                        int64_t batch, int64_t dim, int64_t seqlen, int dstate,
                        ss_dtype in_dtype, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream, const float* conv_w = nullptr,
                        const float* conv_b = nullptr, int conv_width = 0, bool zoh = false,
                        float* ckpt = nullptr) {
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
  if (conv_w && (conv_width < 1 || conv_width > kConvTaps)) return SS_ERR_UNSUPPORTED;
  const void* f_ptrs[8] = {A, D, delta_bias, y_out, last_state_out, h0, conv_w, conv_b};
  for (const void* p : f_ptrs)
    if (p && !aligned(p, 4)) return SS_ERR_INVALID_ARG;

  FwdArgs a;
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.A = A; a.D = D; a.delta_bias = delta_bias;
  a.y = y_out; a.last_state = last_state_out; a.h0 = h0;
  a.conv_w = conv_w; a.conv_b = conv_w ? conv_b : nullptr; a.conv_width = conv_w ? conv_width : 0;
  a.ckpt = ckpt;
  a.batch = batch; a.dim = dim; a.seqlen = seqlen;
  a.softplus = softplus_flag != 0;
  bool vec = ((size_t)seqlen * es) % 16 == 0;
  for (const void* p : in_ptrs)
    if (p && !aligned(p, 16)) vec = false;
  if (!aligned(y_out, 16)) vec = false;
  a.vec = vec ? 1 : 0;

  const bool f32 = in_dtype == SS_F32;
  void* ws = workspace;
  const size_t wsb = workspace_bytes;
  if (conv_w) {
    if (f32) return dispatch_dtype<float, true, false, false>(a, dstate, ws, wsb, stream);
    return dispatch_dtype<__nv_bfloat16, true, false, false>(a, dstate, ws, wsb, stream);
  }
  if (zoh) {
    if (f32) return dispatch_dtype<float, false, true, false>(a, dstate, ws, wsb, stream);
    return dispatch_dtype<__nv_bfloat16, false, true, false>(a, dstate, ws, wsb, stream);
  }
  if (ckpt) {
    if (f32) return dispatch_dtype<float, false, false, true>(a, dstate, ws, wsb, stream);
    return dispatch_dtype<__nv_bfloat16, false, false, true>(a, dstate, ws, wsb, stream);
  }
  if (f32) return dispatch_dtype<float, false, false, false>(a, dstate, ws, wsb, stream);
  return dispatch_dtype<__nv_bfloat16, false, false, false>(a, dstate, ws, wsb, stream);
}

}  // namespace
}  // namespace ssscan

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

ss_status ss_debug_inject(int what, long long value) {
  switch (what) {
    case SS_DEBUG_FORCE_WORKERS: g_dbg_workers.store(value); return SS_OK;
    case SS_DEBUG_SKIP_PUBLISH: g_dbg_skip_publish.store(value); return SS_OK;
    case SS_DEBUG_SPIN_LIMIT: g_dbg_spin_limit.store(value); return SS_OK;
    case SS_DEBUG_STEP_SIMPLE: g_dbg_step_simple.store(value); return SS_OK;
    case SS_DEBUG_CLEAR:
      g_dbg_step_simple.store(0);
      g_dbg_workers.store(0);
      g_dbg_skip_publish.store(-1);
      g_dbg_spin_limit.store(0);
      return SS_OK;
  }
  return SS_ERR_INVALID_ARG;
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
