// scan_fix.cuh -- carry-in correction for a sequence scanned in segments.
//
// A long sequence with few channels is cut into segments that the chunked
// kernel scans at the same time, each from h = 0 (the first from the given
// initial state).  Over segment s the true state is
//     h_t = hl_t + P_t h_in,   P_t[n] = prod_{k = start(s)}^{t} A_bar_k[n]
//                                     = 2^(A[d,n] log2(e) sum_{k <= t} Delta_k),
// where hl is the local state and h_in the state the previous segments end
// in: the linear recurrence composes with the associative operator
// (a, b) then (a', b') = (a' a, a' b + b') ("Mamba 选择性机制", sec. 3.1), so
// h_in follows from the segments' (prod A_bar, end state) pairs.  The local
// readout therefore misses sum_n C_t[n] P_t[n] h_in[n], gated by SiLU(z_t);
// this kernel adds it to y and writes the final state.
//
// One warp per (batch row, channel, segment >= 1).  Each lane takes four
// consecutive steps of every 128-step block; the prefix sums of Delta over the
// segment come from a per-lane sum and a warp scan (the running total in
// double).  The term of state n is evaluated as sign(h_in[n]) 2^(a_n S_t +
// log2|h_in[n]|) C_t[n] (one fused multiply-add for the exponent).  A state's
// term is dropped once |h_in[n]| P_t[n] < 2^-36 max_m |h_in[m]| for the rest of
// the segment: with softplus on (Delta >= 0) and A[d,n] < 0 the weight only
// falls, and a term 2^-36 below the largest state lies 12 binary orders below
// the fp32 resolution of the readout it would be added to.  Otherwise
// (A >= 0, or Delta of either sign) the term is kept for the whole segment.
// The states are visited in the order they are dropped, latest first, so the
// live ones are always a prefix of that order, and the walk ends at the first
// block where none is live.
//
// With 16-byte aligned rows, one lane of the warp brings each block's delta,
// z, y (and, for N = 16, the block's C tile) into shared memory with TMA, two
// blocks deep, completing on a per-warp mbarrier; otherwise the lanes load
// element-wise.
#pragma once

#include "pointwise.cuh"

namespace ssscan {

struct FixArgs {
  const void* delta;
  const void* z;  // nullable
  const void* C;
  const float* A;
  const float* delta_bias;  // nullable
  float* y;
  float* last_state;  // nullable
  const float* seg_h;     // [batch * dim][nseg][N] segment end states
  const float* seg_dsum;  // [batch * dim][nseg] sum of Delta per segment
  int64_t batch, dim, seqlen;
  int64_t seg_len;  // steps per segment, a multiple of 32 (the last may be shorter)
  int nseg;
  int softplus;
  int tma;  // 1: 16-byte aligned rows, the blocks come in by TMA (maps valid)
};

// TMA descriptors of the correction: delta, z and y as [batch][dim][L] with a
// [1][1][128] box, C as [batch][N][L] with a [1][N][128] box (N = 16 only).
struct FixMaps {
  CUtensorMap delta, z, y, C;
};

constexpr int kFixWarps = 4;
constexpr int kFixBlock = 128;         // steps per block (4 per lane)
constexpr float kFixDropLog2 = -36.f;  // log2 of a term's weight, relative to the largest
                                       // state, below which it is dropped

// Per-warp staging of one block (byte offsets, each a multiple of 128).
template <typename Tin, int N>
struct FixStage {
  static constexpr int ES = (int)sizeof(Tin);
  static constexpr bool STAGE_C = N == 16;
  static constexpr int ROW = kFixBlock * ES;  // one 128-step row of an input
  static constexpr int C_BYTES = STAGE_C ? N * ROW : 0;
  static constexpr int D_OFF = C_BYTES;
  static constexpr int Z_OFF = D_OFF + ROW;
  static constexpr int Y_OFF = Z_OFF + ROW;
  static constexpr int BYTES = Y_OFF + kFixBlock * 4;  // one stage
  static constexpr int SMEM = kFixWarps * 2 * BYTES + 128;  // + slack to align the base
  static_assert(ROW % 128 == 0 && BYTES % 128 == 0, "TMA destinations 128-byte aligned");
};

// Four consecutive elements from t (zeros past `end`), widened to float.
// (row_ix: the row's first element index in its tensor of `total` elements)
template <typename T>
__device__ __forceinline__ float4 fix_load4(const T* row, int64_t t, int64_t end, int64_t row_ix,
                                            int64_t total) {
  float e[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    e[k] = (t + k < end && in_range(row_ix + t + k, total)) ? to_f32(row[t + k]) : 0.f;
  return make_float4(e[0], e[1], e[2], e[3]);
}

template <typename T>
__device__ __forceinline__ float4 fix_lds4(const unsigned char* p) {
  if constexpr (sizeof(T) == 4) {
    return *reinterpret_cast<const float4*>(p);
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
  }
}

template <typename Tin, int N>
__global__ void __launch_bounds__(kFixWarps * 32)
    scan_fix_kernel(const FixArgs a, const __grid_constant__ FixMaps maps) {
  using FS = FixStage<Tin, N>;
  __shared__ __align__(16) float4 sh_p[kFixWarps][N];  // {a, a, log2|h_in|, log2|h_in|}
  __shared__ int sh_n[kFixWarps][N];    // state index at each position (slowest decay first)
  __shared__ int sh_neg[kFixWarps][N];  // sign of h_in at each position
  __shared__ float sh_sd[kFixWarps][N];  // the largest sum of Delta at which it is kept
  __shared__ __align__(8) uint64_t fbar[kFixWarps][2];
  extern __shared__ __align__(128) unsigned char fix_dyn[];
  unsigned char* fix_smem = fix_dyn + ((128u - (smem_u32(fix_dyn) & 127u)) & 127u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t per_ch = a.nseg - 1;
  const int64_t task = (int64_t)blockIdx.x * kFixWarps + warp;
  if (task >= a.batch * a.dim * per_ch) return;  // whole warps
  const int64_t bd = task / per_ch;  // flat channel b * dim + d
  const int s = (int)(task - bd * per_ch) + 1;
  const int64_t b = bd / a.dim, d = bd - b * a.dim;
  const int64_t L = a.seqlen;
  const int64_t n_act = a.batch * a.dim * L;  // elements of delta, z and y
  const bool tma = a.tma != 0;

  // h_in of segment s: fold the (prod A_bar, end state) pairs of segments
  // 0 .. s-1 in order; the last segment's task also writes the final state.
  const float* hs = a.seg_h + bd * a.nseg * N;
  const float* ds = a.seg_dsum + bd * a.nseg;
  const float* Ad = a.A + d * N;
  const int64_t n_seg = a.batch * a.dim * a.nseg;  // extents of the segment arrays
  if (!in_range(bd * a.nseg, a.nseg, n_seg) || !in_range(d * N, N, a.dim * N)) return;
  float lh_max = -INFINITY;  // log2 max_n |h_in[n]|
  for (int n = lane; n < N; n += 32) {
    const float an = __ldg(Ad + n) * 1.4426950408889634f;
    float h = hs[n];
    for (int q = 1; q < s; ++q) h = fmaf(ex2_approx(an * ds[q]), h, hs[(int64_t)q * N + n]);
    if (s == a.nseg - 1 && a.last_state && in_range(bd * N + n, a.batch * a.dim * N))
      a.last_state[bd * N + n] = fmaf(ex2_approx(an * ds[s]), h, hs[(int64_t)s * N + n]);
    float lh;  // log2|h_in|: -inf for 0, so that its terms vanish
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lh) : "f"(fabsf(h)));
    sh_p[warp][n] = make_float4(an, an, lh, lh);  // by state for now
    sh_neg[warp][n] = h < 0.f;
    lh_max = fmaxf(lh_max, lh);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lh_max = fmaxf(lh_max, __shfl_xor_sync(kFullMask, lh_max, o));
  // The largest S = sum Delta at which state n's term is kept:
  // a_n S + log2|h_in[n]| >= log2 max|h_in| + kFixDropLog2.  It falls with S
  // only for a_n < 0 with Delta >= 0 (softplus); otherwise it is kept.
  for (int n = lane; n < N; n += 32) {
    const float4 p = sh_p[warp][n];
    const bool decays = a.softplus && p.x < 0.f;
    sh_sd[warp][n] = decays ? (lh_max + kFixDropLog2 - p.z) / p.x : INFINITY;
  }
  __syncwarp();
  // positions: states by that limit, latest first, so that the live states
  // are always a prefix of the positions
  float4 pp[(N + 31) / 32];
  float sdv[(N + 31) / 32];
  int ng[(N + 31) / 32], rk[(N + 31) / 32];
#pragma unroll
  for (int q = 0; q < (N + 31) / 32; ++q) {
    const int n = lane + 32 * q;
    if (n < N) {
      const float sd = sh_sd[warp][n];
      int rank = 0;
      for (int m = 0; m < N; ++m) {
        const float sm = sh_sd[warp][m];
        rank += (sm > sd || (sm == sd && m < n)) ? 1 : 0;
      }
      pp[q] = sh_p[warp][n];
      sdv[q] = sd;
      ng[q] = sh_neg[warp][n];
      rk[q] = rank;
    }
  }
  __syncwarp();
#pragma unroll
  for (int q = 0; q < (N + 31) / 32; ++q) {
    const int n = lane + 32 * q;
    if (n < N) {
      sh_p[warp][rk[q]] = pp[q];
      sh_sd[warp][rk[q]] = sdv[q];
      sh_neg[warp][rk[q]] = ng[q];
      sh_n[warp][rk[q]] = n;
    }
  }
  __syncwarp();
  const Tin* drow = static_cast<const Tin*>(a.delta) + bd * L;
  const Tin* zrow = a.z ? static_cast<const Tin*>(a.z) + bd * L : nullptr;
  const Tin* Cb = static_cast<const Tin*>(a.C) + b * (int64_t)N * L;
  float* yrow = a.y + bd * L;
  const float bias = a.delta_bias ? __ldg(a.delta_bias + d) : 0.f;
  const int64_t t_begin = (int64_t)s * a.seg_len;
  const int64_t t_end = t_begin + a.seg_len < L ? t_begin + a.seg_len : L;
  const int64_t nblk = (t_end - t_begin + kFixBlock - 1) / kFixBlock;
  unsigned char* stage = fix_smem + warp * 2 * FS::BYTES;
  uint64_t* bar = fbar[warp];
  const uint32_t tx = FS::C_BYTES + FS::ROW * (zrow ? 2 : 1) + kFixBlock * 4;
  auto issue = [&](int64_t k) {  // lane 0: the TMA loads of block k into stage k & 1
    unsigned char* st = stage + (k & 1) * FS::BYTES;
    const int32_t t0 = (int32_t)(t_begin + k * kFixBlock);
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bar[k & 1], tx);
    if constexpr (FS::STAGE_C) tma_load_3d(st, &maps.C, &bar[k & 1], t0, 0, (int32_t)b);
    tma_load_3d(st + FS::D_OFF, &maps.delta, &bar[k & 1], t0, (int32_t)d, (int32_t)b);
    if (zrow) tma_load_3d(st + FS::Z_OFF, &maps.z, &bar[k & 1], t0, (int32_t)d, (int32_t)b);
    tma_load_3d(st + FS::Y_OFF, &maps.y, &bar[k & 1], t0, (int32_t)d, (int32_t)b);
  };
  if (tma && lane == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    issue(0);
    if (nblk > 1) issue(1);
  }
  __syncwarp();

  int live = N;        // positions [0, live) may still carry weight
  double carry = 0.0;  // sum of Delta over the blocks before this one
  int64_t k = 0;
  bool ok = true;  // false once a bounded wait has given up (error word set)
  for (; k < nblk; ++k) {
    const int64_t t = t_begin + k * kFixBlock + 4 * lane;
    const unsigned char* cur = stage + (k & 1) * FS::BYTES;
    if (tma) {
      ok = __all_sync(kFullMask, mbar_wait_bounded(&bar[k & 1], (uint32_t)((k >> 1) & 1),
                                                   kTmaSpinLimit));
      if (!ok) break;
    }
    const float4 dl4 = tma ? fix_lds4<Tin>(cur + FS::D_OFF + 4 * lane * FS::ES)
                           : fix_load4(drow, t, t_end, bd * L, n_act);
    const float2 b2 = make_float2(bias, bias);
    float2 x01 = __fadd2_rn(make_float2(dl4.x, dl4.y), b2);
    float2 x23 = __fadd2_rn(make_float2(dl4.z, dl4.w), b2);
    if (a.softplus) {
      x01 = softplus_fast2(x01);
      x23 = softplus_fast2(x23);
    }
    float dl[4] = {x01.x, x01.y, x23.x, x23.y};
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      if (t + kk >= t_end) dl[kk] = 0.f;
    float p[4];
    p[0] = dl[0];
    p[1] = p[0] + dl[1];
    p[2] = p[1] + dl[2];
    p[3] = p[2] + dl[3];
    float incl = p[3];  // inclusive scan of the lane totals
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float v = __shfl_up_sync(kFullMask, incl, o);
      if (lane >= o) incl += v;
    }
    const float excl = incl - p[3];
    float S[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) S[kk] = (float)(carry + (double)(excl + p[kk]));
    const float S_first = __shfl_sync(kFullMask, S[0], 0);
    carry += (double)__shfl_sync(kFullMask, incl, 31);
    // S_first is the block's smallest sum: a position dead now stays dead
    while (live > 0 && S_first > sh_sd[warp][live - 1]) --live;
    if (live == 0) break;
    const float2 S01 = make_float2(S[0], S[1]), S23 = make_float2(S[2], S[3]);
    float2 pos01 = make_float2(0.f, 0.f), pos23 = pos01, neg01 = pos01, neg23 = pos01;
#pragma unroll 4
    for (int i = 0; i < live; ++i) {
      const float4 pr = sh_p[warp][i];
      const float4 c4 = (tma && FS::STAGE_C)
                            ? fix_lds4<Tin>(cur + sh_n[warp][i] * FS::ROW + 4 * lane * FS::ES)
                            : fix_load4(Cb + (int64_t)sh_n[warp][i] * L, t, t_end,
                                        (b * N + sh_n[warp][i]) * L, a.batch * N * L);
      const float2 x01e = __ffma2_rn(S01, make_float2(pr.x, pr.y), make_float2(pr.z, pr.w));
      const float2 x23e = __ffma2_rn(S23, make_float2(pr.x, pr.y), make_float2(pr.z, pr.w));
      const float2 e01 = make_float2(ex2_approx(x01e.x), ex2_approx(x01e.y));
      const float2 e23 = make_float2(ex2_approx(x23e.x), ex2_approx(x23e.y));
      if (sh_neg[warp][i]) {  // warp-uniform
        neg01 = __ffma2_rn(make_float2(c4.x, c4.y), e01, neg01);
        neg23 = __ffma2_rn(make_float2(c4.z, c4.w), e23, neg23);
      } else {
        pos01 = __ffma2_rn(make_float2(c4.x, c4.y), e01, pos01);
        pos23 = __ffma2_rn(make_float2(c4.z, c4.w), e23, pos23);
      }
    }
    const float2 c01 = __fadd2_rn(pos01, make_float2(-neg01.x, -neg01.y));
    const float2 c23 = __fadd2_rn(pos23, make_float2(-neg23.x, -neg23.y));
    const float4 y4 = tma ? fix_lds4<float>(cur + FS::Y_OFF + 16 * lane)
                          : fix_load4(yrow, t, t_end, bd * L, n_act);
    float2 g01 = make_float2(1.f, 1.f), g23 = g01;
    if (zrow) {
      const float4 z4 = tma ? fix_lds4<Tin>(cur + FS::Z_OFF + 4 * lane * FS::ES)
                            : fix_load4(zrow, t, t_end, bd * L, n_act);
      g01 = silu_fast2(make_float2(z4.x, z4.y));
      g23 = silu_fast2(make_float2(z4.z, z4.w));
    }
    const float2 o01 = __ffma2_rn(c01, g01, make_float2(y4.x, y4.y));
    const float2 o23 = __ffma2_rn(c23, g23, make_float2(y4.z, y4.w));
    if (tma && t + 3 < t_end) {
      if (in_range(bd * L + t, 4, n_act))
        *reinterpret_cast<float4*>(yrow + t) = make_float4(o01.x, o01.y, o23.x, o23.y);
    } else {
      const float out[4] = {o01.x, o01.y, o23.x, o23.y};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        if (t + kk < t_end && in_range(bd * L + t + kk, n_act)) yrow[t + kk] = out[kk];
    }
    __syncwarp();  // every lane is done with this stage before TMA refills it
    if (tma && lane == 0 && k + 2 < nblk) issue(k + 2);
  }
  // No copy may land after the warp has left.  Issued: blocks up to k + 1
  // (the loop issues k + 2 only at the end of iteration k).  Waited: up to
  // k - 1, and k itself unless its wait gave up.
  if (tma && lane == 0) {
    const int64_t last = k + 1 < nblk ? k + 1 : nblk - 1;
    for (int64_t kk = ok ? k + 1 : k; kk <= last; ++kk)
      mbar_wait_bounded(&bar[kk & 1], (uint32_t)((kk >> 1) & 1), kTmaSpinLimit);
  }
  __syncwarp();
}

}  // namespace ssscan
