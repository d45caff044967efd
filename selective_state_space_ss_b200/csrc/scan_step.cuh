// scan_step.cuh -- one recurrent (decode) step of the selective SSM.
//
// Inference keeps the state h [batch, dim, N] between tokens and advances it
// one token at a time with O(1) work per token ("从Transformer的痛点说起 ...
// Mamba", sec. 5.1 table and sec. 6.3): for every (b, d) and n,
//   Delta = softplus(delta[b,d] + bias[d]),
//   h[n]  = 2^(Delta A[d,n] log2 e) h[n] + Delta u[b,d] B[b,n],
//   y     = (sum_n C[b,n] h[n] + D[d] u[b,d]) SiLU(z[b,d]),
// with h read and written in place.  Every state element is touched once per
// step, so the kernel is bound by HBM bandwidth: 8 bytes of state traffic per
// (b, d, n) against 4 FMAs and one ex2.
//
// Two kernels, same arithmetic and lane layout (a lane owns four consecutive
// states of one channel: one 16-byte state vector and one 16-byte vector of
// A, so N/4 consecutive lanes share a channel, a warp's state accesses are
// contiguous 512-byte runs, and the readout's lane partials meet by xor
// shuffles inside the warp):
//
//  scan_step_pipe_kernel (16-byte aligned rows, the normal case): persistent
//    CTAs walk tiles of (batch row b, TILE_CH consecutive channels); a
//    producer warp streams each tile's 16 KB of state, its u/delta/z runs and
//    the row's B, C into a ring of shared-memory stages with bulk asynchronous
//    copies completing on "full" mbarriers, several tiles ahead, so the bytes
//    in flight do not cost registers.  The eight compute warps read a stage,
//    store the new state and y straight to HBM and release the stage on its
//    "empty" mbarrier, each warp on its own, so that no CTA-wide barrier holds
//    the fast warps back.  Tiles are ordered channel-tile-major, so a CTA's
//    consecutive tiles share A, D and the bias, which stay in registers.
//    The kernel is launched as a programmatic dependent of the previous
//    kernel in the stream: its CTAs may start and set up their barriers while
//    that kernel drains; every thread then waits for the previous grid to
//    complete (griddepcontrol.wait, which also makes its writes visible)
//    before it reads anything from global memory.  Each CTA in turn lets the
//    next step's grid launch as soon as it starts.
//  scan_step_kernel (any alignment): one batch row per grid row, plain loads.
#pragma once

#include "pointwise.cuh"

namespace ssscan {

struct StepArgs {
  const void* u;      // [batch, dim]
  const void* delta;  // [batch, dim]
  const void* z;      // [batch, dim], nullable
  const void* B;      // [batch, N]
  const void* C;      // [batch, N]
  const float* A;     // [dim, N]
  const float* D;           // [dim], nullable
  const float* delta_bias;  // [dim], nullable
  float* state;             // [batch, dim, N], read and written in place
  float* y;                 // [batch, dim]
  int64_t batch, dim;
  int softplus;
};

constexpr int kStepThreads = 256;
#ifndef SS_STEP_UNITS
#define SS_STEP_UNITS 2
#endif
#ifndef SS_STEP_MIN_BLOCKS
#define SS_STEP_MIN_BLOCKS 4
#endif
constexpr int kStepUnits = SS_STEP_UNITS;  // 4-state vectors per thread, kStepThreads apart

// Four consecutive elements of an input row, widened to float.  kVec: one
// 16-byte (f32) or 8-byte (bf16) load; otherwise four element loads.
template <bool kVec>
__device__ __forceinline__ float4 ld4(const float* p) {
  if constexpr (kVec) return __ldg(reinterpret_cast<const float4*>(p));
  return make_float4(__ldg(p), __ldg(p + 1), __ldg(p + 2), __ldg(p + 3));
}
template <bool kVec>
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  if constexpr (kVec) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
  }
  return make_float4(__bfloat162float(p[0]), __bfloat162float(p[1]), __bfloat162float(p[2]),
                     __bfloat162float(p[3]));
}
// The state may not go through the read-only path: it is written by this
// kernel (the same thread reads, then writes its own vector).
template <bool kVec>
__device__ __forceinline__ float4 ld_state(const float* p) {
  if constexpr (kVec) return *reinterpret_cast<const float4*>(p);
  return make_float4(p[0], p[1], p[2], p[3]);
}
template <bool kVec>
__device__ __forceinline__ void st_state(float* p, float4 v) {
  if constexpr (kVec) {
    *reinterpret_cast<float4*>(p) = v;
  } else {
    p[0] = v.x; p[1] = v.y; p[2] = v.z; p[3] = v.w;
  }
}

template <typename E, int N, bool kVec>
__global__ void __launch_bounds__(kStepThreads, SS_STEP_MIN_BLOCKS)
    scan_step_kernel(const StepArgs a) {
  constexpr int LPC = N / 4;  // lanes per channel
  static_assert(N % 4 == 0 && LPC <= 32 && (32 % LPC) == 0, "lanes of a channel share a warp");
  static_assert(kStepThreads % LPC == 0, "a thread's units share one state vector index j");
  const E* __restrict__ u = static_cast<const E*>(a.u);
  const E* __restrict__ dl = static_cast<const E*>(a.delta);
  const E* __restrict__ zp = static_cast<const E*>(a.z);
  const E* __restrict__ Bp = static_cast<const E*>(a.B);
  const E* __restrict__ Cp = static_cast<const E*>(a.C);
  // 4-state vectors per batch row (the host keeps dim * N below 2^31)
  const int row_units = (int)a.dim * LPC;
  const int j = threadIdx.x % LPC;  // the same for every unit of this thread
  const int base = blockIdx.x * (kStepThreads * kStepUnits) + threadIdx.x;

  for (int64_t b = blockIdx.y; b < a.batch; b += gridDim.y) {
    float* srow = a.state + b * row_units * 4;
    const int64_t crow = b * a.dim;  // first channel of this row
    const float4 bv = ld4<kVec>(Bp + b * N + j * 4);
    const float4 cv = ld4<kVec>(Cp + b * N + j * 4);
    float4 h[kStepUnits], av[kStepUnits];
    float uu[kStepUnits], xx[kStepUnits], zz[kStepUnits], Dd[kStepUnits];
    // all loads first: kStepUnits independent state vectors in flight per thread
#pragma unroll
    for (int k = 0; k < kStepUnits; ++k) {
      const int r = base + k * kStepThreads;
      const int d = r / LPC;
      const bool in = r < row_units && in_range((int64_t)b * row_units + r, a.batch * row_units) &&
                      in_range(crow + d, a.batch * a.dim);
      h[k] = in ? ld_state<kVec>(srow + r * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      av[k] = in ? ld4<kVec>(a.A + r * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      uu[k] = in ? to_f32(u[crow + d]) : 0.f;
      xx[k] = in ? to_f32(dl[crow + d]) + (a.delta_bias ? __ldg(a.delta_bias + d) : 0.f) : 0.f;
      zz[k] = (in && zp) ? to_f32(zp[crow + d]) : 0.f;
      Dd[k] = (in && a.D) ? __ldg(a.D + d) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kStepUnits; ++k) {
      const int r = base + k * kStepThreads;
      const float dt = a.softplus ? softplus_fast(xx[k]) : xx[k];
      const float dtu = dt * uu[k];
      const float s = dt * 1.4426950408889634f;
      h[k].x = fmaf(ex2_approx(s * av[k].x), h[k].x, dtu * bv.x);
      h[k].y = fmaf(ex2_approx(s * av[k].y), h[k].y, dtu * bv.y);
      h[k].z = fmaf(ex2_approx(s * av[k].z), h[k].z, dtu * bv.z);
      h[k].w = fmaf(ex2_approx(s * av[k].w), h[k].w, dtu * bv.w);
      float part = cv.x * h[k].x;
      part = fmaf(cv.y, h[k].y, part);
      part = fmaf(cv.z, h[k].z, part);
      part = fmaf(cv.w, h[k].w, part);
#pragma unroll
      for (int off = LPC / 2; off > 0; off >>= 1) part += __shfl_xor_sync(kFullMask, part, off);
      if (r < row_units && in_range((int64_t)b * row_units + r, a.batch * row_units)) {
        st_state<kVec>(srow + r * 4, h[k]);
        if (j == 0) {
          float y = part + Dd[k] * uu[k];
          if (zp) y *= silu_fast(zz[k]);
          a.y[crow + r / LPC] = y;
        }
      }
    }
  }
}

// ------------------------------------------------ pipelined (bulk copies) ---

#ifndef SS_STEP_PIPE_STAGES
#define SS_STEP_PIPE_STAGES 4
#endif
#ifndef SS_STEP_PIPE_CTAS
#define SS_STEP_PIPE_CTAS 4
#endif
#ifndef SS_STEP_PIPE_UPT
#define SS_STEP_PIPE_UPT 2
#endif

struct StepPipeSched {
  int64_t tiles_per_row;  // channel tiles per batch row
  int64_t items;          // tiles_per_row * batch
};

template <typename E, int N>
struct StepPipeCfg {
  static constexpr int NT = 256;                  // compute threads per CTA
  static constexpr int CWARPS = NT / 32;          // compute warps (arrivals on an empty barrier)
  static constexpr int THREADS = NT + 32;         // + the producer warp
  static constexpr int UPT = SS_STEP_PIPE_UPT;    // 4-state vectors per thread per tile
  static constexpr int LPC = N / 4;               // lanes per channel
  static constexpr int UNITS = NT * UPT;          // 4-state vectors per tile
  static constexpr int TILE_CH = UNITS / LPC;     // channels per tile
  static constexpr int ES = sizeof(E);
  static constexpr int STATE_BYTES = UNITS * 16;
  static constexpr int ACT_BYTES = (TILE_CH * ES + 15) / 16 * 16;
  static constexpr int SEL_BYTES = (N * ES + 15) / 16 * 16;
  static constexpr int OFF_U = STATE_BYTES;
  static constexpr int OFF_DELTA = OFF_U + ACT_BYTES;
  static constexpr int OFF_Z = OFF_DELTA + ACT_BYTES;
  static constexpr int OFF_B = OFF_Z + ACT_BYTES;
  static constexpr int OFF_C = OFF_B + SEL_BYTES;
  static constexpr int STAGE = (OFF_C + SEL_BYTES + 127) / 128 * 128;
  static constexpr int STAGES = SS_STEP_PIPE_STAGES;
  static constexpr int SMEM_BYTES = STAGES * STAGE + 128;  // + alignment slack
  static_assert(NT % LPC == 0, "a thread's units share one state vector index j");
  static_assert((TILE_CH * ES) % 16 == 0, "bulk copies of whole tiles are 16-byte multiples");
};

template <typename E, int N>
__global__ void __launch_bounds__(StepPipeCfg<E, N>::THREADS, SS_STEP_PIPE_CTAS)
    scan_step_pipe_kernel(const StepArgs a, const StepPipeSched sc) {
  using CF = StepPipeCfg<E, N>;
  constexpr int LPC = CF::LPC, UPT = CF::UPT, S = CF::STAGES;
  extern __shared__ __align__(128) unsigned char smem_dyn[];
  unsigned char* smem = smem_dyn + ((128u - (smem_u32(smem_dyn) & 127u)) & 127u);
  __shared__ __align__(8) uint64_t full[S];   // stage holds its tile (1 arrival + bytes)
  __shared__ __align__(8) uint64_t empty[S];  // every compute warp is done with the stage

  const int w = blockIdx.x;
  const int64_t i0 = sc.items * w / gridDim.x, i1 = sc.items * (w + 1) / gridDim.x;
  const int64_t n = i1 - i0;
  const int tid = threadIdx.x;
  const int j = tid % LPC;
  const bool has_z = a.z != nullptr;
  const E* u = static_cast<const E*>(a.u);
  const E* dl = static_cast<const E*>(a.delta);
  const E* zp = static_cast<const E*>(a.z);
  const E* Bp = static_cast<const E*>(a.B);
  const E* Cp = static_cast<const E*>(a.C);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CF::CWARPS);
    }
    fence_mbar_init();
    // the next kernel in the stream may be scheduled once every CTA of this
    // grid has started (it waits for this grid's completion before its reads)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  __syncthreads();
  if (n <= 0) return;

  // item i -> (channel tile c, batch row b), c-major; the producer walks its
  // own copy of the cursor up to S items ahead of the compute warps
  auto seat = [&](int64_t i, int64_t& c, int64_t& b) {
    c = i / a.batch;
    b = i - c * a.batch;
  };
  auto issue = [&](int64_t k, int64_t c, int64_t b) {  // item i0 + k into stage k % S
    unsigned char* st = smem + (k % S) * CF::STAGE;
    const int64_t d0 = c * CF::TILE_CH;
    const int64_t nch = a.dim - d0 < CF::TILE_CH ? a.dim - d0 : CF::TILE_CH;
    const uint32_t sb = (uint32_t)(nch * N * 4), ab = (uint32_t)(nch * CF::ES);
    const uint32_t tx = sb + (has_z ? 3u : 2u) * ab + 2u * N * CF::ES;
    const int64_t ch0 = b * a.dim + d0;
    // (checked builds: the copied ranges lie inside their tensors, else nothing is copied)
    if (!in_range(ch0 * N, nch * N, a.batch * a.dim * N) || !in_range(ch0, nch, a.batch * a.dim) ||
        !in_range(b * N, N, a.batch * N))
      return;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&full[k % S], tx);
    bulk_load(st, a.state + ch0 * N, sb, &full[k % S]);
    bulk_load(st + CF::OFF_U, u + ch0, ab, &full[k % S]);
    bulk_load(st + CF::OFF_DELTA, dl + ch0, ab, &full[k % S]);
    if (has_z) bulk_load(st + CF::OFF_Z, zp + ch0, ab, &full[k % S]);
    bulk_load(st + CF::OFF_B, Bp + b * N, N * CF::ES, &full[k % S]);
    bulk_load(st + CF::OFF_C, Cp + b * N, N * CF::ES, &full[k % S]);
  };

  if (tid >= CF::NT) {  // the producer warp: one lane issues, the rest leave
    if (tid == CF::NT) {
      // every read below may see writes of the previous kernel in the stream
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int64_t pc, pb;
      seat(i0, pc, pb);
      int64_t k = 0;
      for (; k < n; ++k) {
        // stage k % S is free once every compute warp has released item k - S
        if (k >= S &&
            !mbar_wait_bounded(&empty[k % S], (uint32_t)((k / S - 1) & 1), kTmaSpinLimit))
          break;
        issue(k, pc, pb);
        if (++pb == a.batch) { pb = 0; ++pc; }
      }
      // no copy may land after the CTA has left: wait (bounded) for the last
      // S items issued (the earlier ones were released, so they have landed)
      for (int64_t kk = k > S ? k - S : 0; kk < k; ++kk)
        mbar_wait_bounded(&full[kk % S], (uint32_t)((kk / S) & 1), kTmaSpinLimit);
    }
    return;
  }

  asm volatile("griddepcontrol.wait;" ::: "memory");  // as the producer's
  int64_t c, b;
  seat(i0, c, b);
  int64_t c_regs = -1;  // channel tile whose A, D, bias sit in registers
  float4 av[UPT];
  float Dd[UPT], bias[UPT];
  for (int64_t k = 0; k < n; ++k) {
    if (c != c_regs) {
#pragma unroll
      for (int q = 0; q < UPT; ++q) {
        const int unit = tid + q * CF::NT;
        const int64_t d = c * CF::TILE_CH + unit / LPC;
        const bool in = d < a.dim && in_range(d * N + 4 * j, 4, a.dim * N);
        const float4 A4 = in ? __ldg(reinterpret_cast<const float4*>(a.A + d * N + 4 * j))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        av[q] = make_float4(A4.x * 1.4426950408889634f, A4.y * 1.4426950408889634f,
                            A4.z * 1.4426950408889634f, A4.w * 1.4426950408889634f);
        Dd[q] = (in && a.D) ? __ldg(a.D + d) : 0.f;
        bias[q] = (in && a.delta_bias) ? __ldg(a.delta_bias + d) : 0.f;
      }
      c_regs = c;
    }
    // a copy that never completes ends this warp; the producer then stops at
    // its next bounded wait for this warp's release and drains its copies
    if (!__all_sync(kFullMask, mbar_wait_bounded(&full[k % S], (uint32_t)((k / S) & 1),
                                                 kTmaSpinLimit)))
      return;
    const unsigned char* st = smem + (k % S) * CF::STAGE;
    const E* su = reinterpret_cast<const E*>(st + CF::OFF_U);
    const E* sd = reinterpret_cast<const E*>(st + CF::OFF_DELTA);
    const E* sz = reinterpret_cast<const E*>(st + CF::OFF_Z);
    const float4 bv = load4_f32(reinterpret_cast<const E*>(st + CF::OFF_B) + 4 * j);
    const float4 cv = load4_f32(reinterpret_cast<const E*>(st + CF::OFF_C) + 4 * j);
    const int64_t ch0 = b * a.dim + c * CF::TILE_CH;
#pragma unroll
    for (int q = 0; q < UPT; ++q) {
      const int unit = tid + q * CF::NT;
      const int cl = unit / LPC;
      float4 h = reinterpret_cast<const float4*>(st)[unit];
      const float uu = to_f32(su[cl]);
      const float x = to_f32(sd[cl]) + bias[q];
      const float dt = a.softplus ? softplus_fast(x) : x;
      const float dtu = dt * uu;
      h.x = fmaf(ex2_approx(dt * av[q].x), h.x, dtu * bv.x);
      h.y = fmaf(ex2_approx(dt * av[q].y), h.y, dtu * bv.y);
      h.z = fmaf(ex2_approx(dt * av[q].z), h.z, dtu * bv.z);
      h.w = fmaf(ex2_approx(dt * av[q].w), h.w, dtu * bv.w);
      float part = cv.x * h.x;
      part = fmaf(cv.y, h.y, part);
      part = fmaf(cv.z, h.z, part);
      part = fmaf(cv.w, h.w, part);
#pragma unroll
      for (int off = LPC / 2; off > 0; off >>= 1) part += __shfl_xor_sync(kFullMask, part, off);
      if (c * CF::TILE_CH + cl < a.dim && in_range((ch0 + cl) * N + 4 * j, 4, a.batch * a.dim * N)) {
        *reinterpret_cast<float4*>(a.state + (ch0 + cl) * N + 4 * j) = h;
        if (j == 0) {
          float y = part + Dd[q] * uu;
          if (has_z) y *= silu_fast(to_f32(sz[cl]));
          a.y[ch0 + cl] = y;
        }
      }
    }
    __syncwarp();  // the warp's lanes are done with stage k % S
    if ((tid & 31) == 0) mbar_arrive(&empty[k % S]);
    if (++b == a.batch) { b = 0; ++c; }
  }
}

}  // namespace ssscan
