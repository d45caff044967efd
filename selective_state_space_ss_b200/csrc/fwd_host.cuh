// fwd_host.cuh -- host side of the forward scan: TMA descriptors, the
// schedule plan (balanced workers or sequence segments), launches and the
// argument checks behind ss_scan_fwd and its variants
// (host code of libssscan.so; the library is one translation unit, ss_scan.cu)
#pragma once

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <chrono>
#include <climits>
#include <cstdint>
#include <cstring>

#include "ss_scan.h"
#include "host_common.cuh"
#include "scan_fwd_chunked.cuh"
#include "scan_fix.cuh"

namespace ssscan {
namespace {

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

constexpr uint32_t kCarrySpinLimit = 1u << 22;  // ~1 s of polling with back-off

// A launch-unique 64-bit epoch: carry flags written by earlier launches (or
// arbitrary bytes in a fresh workspace) never equal it.
unsigned long long next_epoch() {
  static std::atomic<unsigned long long> ctr{
      (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() *
      0x9E3779B97F4A7C15ULL};
  return ctr.fetch_add(0x9E3779B97F4A7C15ULL) | 1ULL;
}

// How the work is cut: `workers` CTAs, each an equal contiguous range of
// (channel group, chunk) units.  workers == groups means one group per CTA and
// no carries; fewer workers balance the load across SMs with carry handoff.
// With fewer channel groups than resident CTA slots (a long sequence over few
// channels), the plain schedule cuts each group's chunks into `nseg` segments
// scanned at once; a second kernel then adds each segment's carry-in.
struct Plan {
  int workers = 0;
  int64_t groups = 0, nk = 0, tiles = 0;
  int nseg = 1;
  int64_t seg_chunks = 0;
  size_t carry_bytes = 0, flag_bytes = 0, seg_h_bytes = 0, ws_bytes = 0;
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
    p->flag_bytes = align256((size_t)p->workers * sizeof(unsigned long long));
    p->ws_bytes = p->carry_bytes + p->flag_bytes + 256;  // + the worker ticket counter
    return true;
  }
  // Segments: fill the resident slots once (groups x nseg CTAs).  Not for the
  // training variant, whose checkpoints must hold true states.
  int64_t nseg = 1;
  const bool can_segment = !CF::TRAIN && CF::WT == 1;
  if (can_segment && forced <= 0 && p->groups < slots) nseg = slots / p->groups;
  const long long fseg = g_dbg_segments.load();
  if (fseg > 0 && can_segment) nseg = fseg;
  if (nseg > p->nk) nseg = p->nk;
  if (nseg > 1) {
    p->seg_chunks = (p->nk + nseg - 1) / nseg;
    nseg = (p->nk + p->seg_chunks - 1) / p->seg_chunks;  // no empty segment
  }
  if (nseg > 1) {
    if (p->groups * nseg > INT_MAX) return false;
    p->nseg = (int)nseg;
    const size_t chans = (size_t)(p->groups * CF::CH);  // >= batch * dim
    p->seg_h_bytes = align256(chans * (size_t)nseg * CF::N * sizeof(float));
    p->ws_bytes = p->seg_h_bytes + align256(chans * (size_t)nseg * sizeof(float));
  } else {
    p->nseg = 1;
    p->seg_chunks = p->nk;
  }
  return true;
}

template <typename E, int N>
struct FixTag {};  // one once-per-device cache per correction kernel

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
  sc.ticket = nullptr;
  const long long spin = g_dbg_spin_limit.exchange(0);
  sc.spin_limit = spin > 0 ? (uint32_t)spin : kCarrySpinLimit;
  sc.skip_publish = (int)g_dbg_skip_publish.exchange(-1);
  sc.nseg = p.nseg;
  sc.seg_chunks = p.seg_chunks;
  g_dbg_workers.store(0);
  g_dbg_segments.store(0);
  if (p.workers < p.groups) {
    // worker ids come from a counter taken at CTA start, so a worker's
    // predecessor is always already resident; the counter starts at 0 per launch
    sc.ticket = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + p.carry_bytes +
                                                p.flag_bytes);
    if (cudaMemsetAsync(sc.ticket, 0, sizeof(unsigned int), stream) != cudaSuccess)
      return SS_ERR_CUDA;
    scan_fwd_chunked_kernel<CF, true><<<(unsigned)p.workers, CF::NT, CF::SMEM_BYTES, stream>>>(a, maps, sc);
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
  }
  if (p.nseg > 1) {
    a.seg_h = static_cast<float*>(workspace);
    a.seg_dsum = reinterpret_cast<float*>(static_cast<char*>(workspace) + p.seg_h_bytes);
  }
  scan_fwd_chunked_kernel<CF, false>
      <<<(unsigned)(p.groups * p.nseg), CF::NT, CF::SMEM_BYTES, stream>>>(a, maps, sc);
  if (cudaGetLastError() != cudaSuccess) return SS_ERR_CUDA;
  if (p.nseg == 1) return SS_OK;
  FixArgs f;
  f.delta = a.delta; f.z = a.z; f.C = a.C; f.A = a.A; f.delta_bias = a.delta_bias;
  f.y = a.y; f.last_state = a.last_state; f.seg_h = a.seg_h; f.seg_dsum = a.seg_dsum;
  f.batch = a.batch; f.dim = a.dim; f.seqlen = a.seqlen;
  f.seg_len = p.seg_chunks * CF::T;
  f.nseg = p.nseg;
  f.softplus = a.softplus;
  using E = typename CF::Elem;
  using FS = FixStage<E, CF::N>;
  const bool bf16 = sizeof(E) == 2;
  FixMaps fm;
  memset(&fm, 0, sizeof fm);
  // TMA blocks need the forward's 16-byte aligned rows (a.vec)
  f.tma = a.vec && encode_3d(&fm.delta, a.delta, bf16, a.seqlen, a.dim, a.batch, FS::BLOCK, 1) &&
          encode_3d(&fm.z, a.z ? a.z : a.delta, bf16, a.seqlen, a.dim, a.batch, FS::BLOCK, 1) &&
          encode_3d(&fm.y, a.y, false, a.seqlen, a.dim, a.batch, FS::BLOCK, 1) &&
          (!FS::STAGE_C || encode_3d(&fm.C, a.C, bf16, a.seqlen, CF::N, a.batch, FS::BLOCK, CF::N));
  const int64_t tasks = a.batch * a.dim * (p.nseg - 1);
  const int64_t blocks = (tasks + kFixWarps - 1) / kFixWarps;
  if (blocks > INT_MAX) return SS_ERR_INVALID_ARG;
  if (once_per_device<FixTag<E, CF::N>>([] {
        return cudaFuncSetAttribute(scan_fix_kernel<E, CF::N, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    FS::SMEM) == cudaSuccess &&
               cudaFuncSetAttribute(scan_fix_kernel<E, CF::N, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    FS::SMEM) == cudaSuccess;
      }) != 1)
    return SS_ERR_CUDA;
  if (f.tma)
    scan_fix_kernel<E, CF::N, true><<<(unsigned)blocks, kFixWarps * 32, FS::SMEM, stream>>>(f, fm);
  else
    scan_fix_kernel<E, CF::N, false><<<(unsigned)blocks, kFixWarps * 32, 0, stream>>>(f, fm);
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

// Channels per lane of the plain forward at N = 16 (the variants use one).
#ifndef SS_N16_CPL
#define SS_N16_CPL 1
#endif
template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Cfg16 = ChunkedCfg<E, 16, SS_N16_K, SS_N16_W, SS_N16_T, (CV || Z || TR) ? 1 : SS_N16_CPL,
                         CV, Z, TR>;
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

// Time-split shapes for short sequences over too few channels to fill the GPU:
// one warp's worth of channels (8) per CTA, 8 warps splitting each chunk in
// time, joined inside the CTA.  (Long sequences are cut into segments instead,
// whose carry-in correction is a second pass; over a short sequence that pass
// would cost about as much as the scan.)
template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Split16 = ChunkedCfg<E, 16, 4, 8, 128, 1, CV, Z, TR, 8>;
template <typename E, bool CV = false, bool Z = false, bool TR = false>
using Split32 = ChunkedCfg<E, 32, 4, 8, 32, 1, CV, Z, TR, 8>;
constexpr int64_t kSplitMaxSeq = 65536;  // longer sequences take segments

// The time split for this shape (not when a test forces segments).
template <class CF>
bool use_time_split(int64_t batch, int64_t dim, int64_t seqlen) {
  if (g_dbg_segments.load() > 0 || seqlen >= kSplitMaxSeq) return false;
  const int64_t groups = batch * ((dim + CF::CH - 1) / CF::CH);
  return groups < device_sms();
}

template <typename E, bool CV, bool Z, bool TR>
ss_status dispatch_dtype(const FwdArgs& a, int N, void* ws, size_t wsb, cudaStream_t stream) {
  switch (N) {
    case 16:
      if (use_time_split<Cfg16<E, CV, Z, TR>>(a.batch, a.dim, a.seqlen))
        return launch_chunked<Split16<E, CV, Z, TR>>(a, ws, wsb, stream);
      return launch_chunked<Cfg16<E, CV, Z, TR>>(a, ws, wsb, stream);
    case 32:
      if (use_time_split<Cfg32<E, CV, Z, TR>>(a.batch, a.dim, a.seqlen))
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
      ok = use_time_split<Cfg16<E, CV, Z, TR>>(batch, dim, seqlen)
               ? make_plan<Split16<E, CV, Z, TR>>(batch, dim, seqlen, &p)
               : make_plan<Cfg16<E, CV, Z, TR>>(batch, dim, seqlen, &p);
      break;
    case 32:
      ok = use_time_split<Cfg32<E, CV, Z, TR>>(batch, dim, seqlen)
               ? make_plan<Split32<E, CV, Z, TR>>(batch, dim, seqlen, &p)
               : make_plan<Cfg32<E, CV, Z, TR>>(batch, dim, seqlen, &p);
      break;
    case 64: ok = make_plan<Cfg64<E, CV, Z, TR>>(batch, dim, seqlen, &p); break;
    case 128: ok = make_plan<Cfg128<E, CV, Z, TR>>(batch, dim, seqlen, &p); break;
  }
  *bytes = p.ws_bytes;
  return ok;
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
  a.seg_h = nullptr; a.seg_dsum = nullptr;
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
