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
// double).  A state's term is dropped once its weight P is below 2^-40 for the
// rest of the segment: with softplus on (Delta >= 0) and A[d,n] < 0 the weight
// only falls, and 2^-40 |h_in| lies 16 binary orders below the fp32
// resolution of the state it would be added to.  Otherwise (A >= 0, or Delta
// of either sign) the term is kept for the whole segment.  The states are
// visited slowest decay first, so the live ones are always a prefix of that
// order, and the walk ends at the first block where none is live.
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
  int64_t seg_len;  // steps per segment, a multiple of 4 (the last may be shorter)
  int nseg;
  int softplus;
  int vec;  // 1: rows of delta, z, C and y start 16-byte aligned every 4 steps
};

constexpr int kFixWarps = 4;
constexpr float kFixDropLog2 = -40.f;  // log2 of the weight below which a term is dropped
constexpr int kFixBatch = 16;          // C rows loaded together

// Four consecutive elements from t (zeros past `end`), widened to float.
template <typename T>
__device__ __forceinline__ float4 fix_load4(const T* row, int64_t t, int64_t end, bool vec) {
  if (vec && t + 3 < end) {
    if constexpr (sizeof(T) == 4) {
      return *reinterpret_cast<const float4*>(row + t);
    } else {
      const uint2 v = *reinterpret_cast<const uint2*>(row + t);
      return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                         __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    }
  }
  float e[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) e[k] = t + k < end ? to_f32(row[t + k]) : 0.f;
  return make_float4(e[0], e[1], e[2], e[3]);
}

template <typename Tin, int N>
__global__ void __launch_bounds__(kFixWarps * 32) scan_fix_kernel(const FixArgs a) {
  __shared__ float sh_h[kFixWarps][N];  // h_in per state, slowest decay first
  __shared__ float sh_a[kFixWarps][N];  // A log2 e per state, same order
  __shared__ int sh_n[kFixWarps][N];    // the state index of each position
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t per_ch = a.nseg - 1;
  const int64_t task = (int64_t)blockIdx.x * kFixWarps + warp;
  if (task >= a.batch * a.dim * per_ch) return;  // whole warps
  const int64_t bd = task / per_ch;  // flat channel b * dim + d
  const int s = (int)(task - bd * per_ch) + 1;
  const int64_t b = bd / a.dim, d = bd - b * a.dim;
  const int64_t L = a.seqlen;
  const bool vec = a.vec != 0;

  // h_in of segment s: fold the (prod A_bar, end state) pairs of segments
  // 0 .. s-1 in order; the last segment's task also writes the final state.
  // Position of state n: its rank by A log2 e, largest (slowest decay) first.
  const float* hs = a.seg_h + bd * a.nseg * N;
  const float* ds = a.seg_dsum + bd * a.nseg;
  const float* Ad = a.A + d * N;
  for (int n = lane; n < N; n += 32) {
    const float an = __ldg(Ad + n) * 1.4426950408889634f;
    float h = hs[n];
    for (int q = 1; q < s; ++q) h = fmaf(ex2_approx(an * ds[q]), h, hs[(int64_t)q * N + n]);
    if (s == a.nseg - 1 && a.last_state)
      a.last_state[bd * N + n] = fmaf(ex2_approx(an * ds[s]), h, hs[(int64_t)s * N + n]);
    int rank = 0;
    for (int m = 0; m < N; ++m) {
      const float am = __ldg(Ad + m) * 1.4426950408889634f;
      rank += (am > an || (am == an && m < n)) ? 1 : 0;
    }
    sh_h[warp][rank] = h;
    sh_a[warp][rank] = an;
    sh_n[warp][rank] = n;
  }
  __syncwarp();

  const Tin* drow = static_cast<const Tin*>(a.delta) + bd * L;
  const Tin* zrow = a.z ? static_cast<const Tin*>(a.z) + bd * L : nullptr;
  const Tin* Cb = static_cast<const Tin*>(a.C) + b * (int64_t)N * L;
  float* yrow = a.y + bd * L;
  const float bias = a.delta_bias ? __ldg(a.delta_bias + d) : 0.f;
  const int64_t t_begin = (int64_t)s * a.seg_len;
  const int64_t t_end = t_begin + a.seg_len < L ? t_begin + a.seg_len : L;
  int live = N;        // positions [0, live) may still carry weight
  double carry = 0.0;  // sum of Delta over the blocks before this one
  float4 dl4 = fix_load4(drow, t_begin + 4 * lane, t_end, vec);
  for (int64_t t0 = t_begin; t0 < t_end; t0 += 128) {
    const int64_t t = t0 + 4 * lane;
    // this block's z and y (used at its end), the next block's delta
    const float4 z4 = zrow ? fix_load4(zrow, t, t_end, vec) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 y4 = fix_load4(yrow, t, t_end, vec);
    const float4 dn4 = fix_load4(drow, t + 128, t_end, vec);
    float dl[4] = {dl4.x + bias, dl4.y + bias, dl4.z + bias, dl4.w + bias};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (a.softplus) dl[k] = softplus_fast(dl[k]);
      if (t + k >= t_end) dl[k] = 0.f;
    }
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
    for (int k = 0; k < 4; ++k) S[k] = (float)(carry + (double)(excl + p[k]));
    const float S_first = __shfl_sync(kFullMask, S[0], 0);
    carry += (double)__shfl_sync(kFullMask, incl, 31);
    // S_first is the block's smallest sum: a position dead now stays dead
    if (a.softplus)
      while (live > 0 && sh_a[warp][live - 1] < 0.f && sh_a[warp][live - 1] * S_first < kFixDropLog2)
        --live;
    if (live == 0) break;
    float corr[4] = {0.f, 0.f, 0.f, 0.f};
    // the live states' C in groups of kFixBatch, every load of a group issued
    // before the first is used (one L2 round trip per group, not per state)
    for (int i0 = 0; i0 < live; i0 += kFixBatch) {
      float4 c4[kFixBatch];
#pragma unroll
      for (int i = 0; i < kFixBatch; ++i)
        c4[i] = i0 + i < live ? fix_load4(Cb + (int64_t)sh_n[warp][i0 + i] * L, t, t_end, vec)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < kFixBatch; ++i) {
        if (i0 + i < live) {
          const float an = sh_a[warp][i0 + i], hn = sh_h[warp][i0 + i];
          const float cv[4] = {c4[i].x, c4[i].y, c4[i].z, c4[i].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) corr[k] = fmaf(cv[k] * hn, ex2_approx(an * S[k]), corr[k]);
        }
      }
    }
    const float zz[4] = {z4.x, z4.y, z4.z, z4.w};
    const float yy[4] = {y4.x, y4.y, y4.z, y4.w};
    float out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) out[k] = fmaf(corr[k], zrow ? silu_fast(zz[k]) : 1.f, yy[k]);
    if (vec && t + 3 < t_end) {
      *reinterpret_cast<float4*>(yrow + t) = make_float4(out[0], out[1], out[2], out[3]);
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (t + k < t_end) yrow[t + k] = out[k];
    }
    dl4 = dn4;
  }
}

}  // namespace ssscan
