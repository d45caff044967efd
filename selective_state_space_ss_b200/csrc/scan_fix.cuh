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
// One warp per (batch row, channel, segment >= 1).  Each lane takes SPL
// consecutive steps of every block of 32 SPL steps; the prefix sums of Delta
// over the segment come from a per-lane sum and a warp scan, the running
// total kept as an unevaluated sum of two floats (Knuth's two-sum), so that
// it does not drift over a long segment.  The term of state n is evaluated
// as sign(h_in[n]) 2^(a_n S_t + log2|h_in[n]|) C_t[n] (one fused
// multiply-add for the exponent).  A state's
// term is dropped once |h_in[n]| P_t[n] < 2^-36 max_m |h_in[m]| for the rest of
// the segment: with softplus on (Delta >= 0) and A[d,n] < 0 the weight only
// falls, and a term 2^-36 below the largest state lies 12 binary orders below
// the fp32 resolution of the readout it would be added to.  Otherwise
// (A >= 0, or Delta of either sign) the term is kept for the whole segment.
// The states are visited in the order they are dropped, latest first, so the
// live ones are always a prefix of that order, and the walk ends at the first
// block where none is live.
//
// With 16-byte aligned rows, four lanes of the warp bring each block's delta,
// z, y (and, for N = 16, the block's C tile) into shared memory with TMA, two
// blocks deep, completing on a per-warp mbarrier; otherwise the lanes load
// element-wise.  A staged C value takes the sign of h_in[n] by an xor of its
// sign bit as it is read, so that each term is one fused multiply-add.
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
// [1][1][block] box, C as [batch][N][L] with a [1][N][block] box (N = 16
// only); a block is 32 SPL steps (FixStage).
struct FixMaps {
  CUtensorMap delta, z, y, C;
};

// One warp (one task) per CTA: tasks differ in length by orders of magnitude
// (a state's term lives for ~1/(Delta |A|) steps), and a CTA holds its
// resources until its longest warp is done.  Measured on B1 L1048576 D1536
// N16: 1, 2 and 4 warps per CTA take 2.87, 2.97 and 3.01 ms.
constexpr int kFixWarps = 1;
constexpr float kFixDropLog2 = -36.f;  // log2 of a term's weight, relative to the largest
                                       // state, below which it is dropped

// Per-warp staging of one block (byte offsets, each a multiple of 128).
// SPL consecutive steps per lane: 8 for bf16 (the per-position loads and
// the block's fixed work are spread over more steps: 2.68 against 2.87 ms
// with 4 on the workload above), 4 for fp32 (half the staging per step).
template <typename Tin, int N>
struct FixStage {
  static constexpr int ES = (int)sizeof(Tin);
  static constexpr int SPL = ES == 2 ? 8 : 4;
  static constexpr int BLOCK = 32 * SPL;  // steps per block
  static constexpr bool STAGE_C = N == 16;
  static constexpr int ROW = BLOCK * ES;  // one block-long row of an input
  static constexpr int C_BYTES = STAGE_C ? N * ROW : 0;
  static constexpr int D_OFF = C_BYTES;
  static constexpr int Z_OFF = D_OFF + ROW;
  static constexpr int Y_OFF = Z_OFF + ROW;
  static constexpr int BYTES = Y_OFF + BLOCK * 4;  // one stage
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

// Four staged elements widened to float, their sign bits flipped by `flip`
// (0, or the sign bits of every element of a 32-bit word).
template <typename T>
__device__ __forceinline__ float4 fix_lds4x(const unsigned char* p, uint32_t flip) {
  if constexpr (sizeof(T) == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    return make_float4(__uint_as_float(v.x ^ flip), __uint_as_float(v.y ^ flip),
                       __uint_as_float(v.z ^ flip), __uint_as_float(v.w ^ flip));
  } else {
    uint2 v = *reinterpret_cast<const uint2*>(p);
    v.x ^= flip;
    v.y ^= flip;
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
  }
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

// TMA: the blocks come in by TMA (a.tma set); otherwise the lanes load them
// element-wise.  A template parameter, so that neither path's code sits,
// predicated off, in the other's loops.
template <typename Tin, int N, bool TMA>
__global__ void __launch_bounds__(kFixWarps * 32)
    scan_fix_kernel(const FixArgs a, const __grid_constant__ FixMaps maps) {
  using FS = FixStage<Tin, N>;
  __shared__ __align__(16) float4 sh_p[kFixWarps][N];  // {a, a, log2|h_in|, log2|h_in|}
  // {state index, sign bits of h_in < 0 for a 32-bit word of C} at each position
  __shared__ int2 sh_nq[kFixWarps][N];
  constexpr int kFlip = sizeof(Tin) == 2 ? (int)0x80008000u : (int)0x80000000u;
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
  constexpr bool tma = TMA;

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
    sh_nq[warp][n] = make_int2(n, h < 0.f ? kFlip : 0);
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
      ng[q] = sh_nq[warp][n].y;
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
      sh_nq[warp][rk[q]] = make_int2(n, ng[q]);
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
  const int64_t nblk = (t_end - t_begin + FS::BLOCK - 1) / FS::BLOCK;
  unsigned char* stage = fix_smem + warp * 2 * FS::BYTES;
  uint64_t* bar = fbar[warp];
  int live = N;  // positions [0, live) may still carry weight
  const uint32_t tx = FS::C_BYTES + FS::ROW * (zrow ? 2 : 1) + FS::BLOCK * 4;
  // The TMA loads of block k into stage k & 1, after lane 0 has armed the
  // barrier with their bytes: lanes 28..31 the [N][block] tile of C (N = 16),
  // delta, z and y.  Called by the whole warp.
  auto issue = [&](int64_t k) {
    unsigned char* st = stage + (k & 1) * FS::BYTES;
    const int32_t t0 = (int32_t)(t_begin + k * FS::BLOCK);
    if (lane == 0) mbar_arrive_expect_tx(&bar[k & 1], tx);
    __syncwarp();
    if (lane >= 28) {
      fence_proxy_async_smem();
      if (FS::STAGE_C && lane == 28) tma_load_3d(st, &maps.C, &bar[k & 1], t0, 0, (int32_t)b);
      if (lane == 29) tma_load_3d(st + FS::D_OFF, &maps.delta, &bar[k & 1], t0, (int32_t)d, (int32_t)b);
      if (lane == 30 && zrow) tma_load_3d(st + FS::Z_OFF, &maps.z, &bar[k & 1], t0, (int32_t)d, (int32_t)b);
      if (lane == 31) tma_load_3d(st + FS::Y_OFF, &maps.y, &bar[k & 1], t0, (int32_t)d, (int32_t)b);
    }
  };
  if (tma) {
    if (lane == 0) {
      mbar_init(&bar[0], 1);
      mbar_init(&bar[1], 1);
      fence_mbar_init();
    }
    __syncwarp();
    issue(0);
    if (nblk > 1) issue(1);
  }
  __syncwarp();

  // sum of Delta over the blocks before this one: c_hi + c_lo
  float c_hi = 0.f, c_lo = 0.f;
  int64_t k = 0;
  bool ok = true;  // false once a bounded wait has given up (error word set)
  constexpr int SP = FS::SPL, SP2 = SP / 2, SP4 = SP / 4;
  static_assert(SP % 4 == 0, "whole quads per lane");
  for (; k < nblk; ++k) {
    const int64_t t = t_begin + k * FS::BLOCK + SP * lane;
    const unsigned char* cur = stage + (k & 1) * FS::BYTES;
    if (tma) {
      ok = __all_sync(kFullMask, mbar_wait_bounded(&bar[k & 1], (uint32_t)((k >> 1) & 1),
                                                   kTmaSpinLimit));
      if (!ok) break;
    }
    float dl[SP];
    const float2 b2 = make_float2(bias, bias);
#pragma unroll
    for (int q = 0; q < SP4; ++q) {
      const float4 dl4 = tma ? fix_lds4<Tin>(cur + FS::D_OFF + (SP * lane + 4 * q) * FS::ES)
                             : fix_load4(drow, t + 4 * q, t_end, bd * L, n_act);
      float2 x01 = __fadd2_rn(make_float2(dl4.x, dl4.y), b2);
      float2 x23 = __fadd2_rn(make_float2(dl4.z, dl4.w), b2);
      if (a.softplus) {
        x01 = softplus_fast2(x01);
        x23 = softplus_fast2(x23);
      }
      dl[4 * q] = x01.x;
      dl[4 * q + 1] = x01.y;
      dl[4 * q + 2] = x23.x;
      dl[4 * q + 3] = x23.y;
    }
#pragma unroll
    for (int kk = 0; kk < SP; ++kk)
      if (t + kk >= t_end) dl[kk] = 0.f;
    float p[SP];
    p[0] = dl[0];
#pragma unroll
    for (int kk = 1; kk < SP; ++kk) p[kk] = p[kk - 1] + dl[kk];
    float incl = p[SP - 1];  // inclusive scan of the lane totals
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float v = __shfl_up_sync(kFullMask, incl, o);
      if (lane >= o) incl += v;
    }
    const float excl = incl - p[SP - 1];
    float2 S2[SP2];
#pragma unroll
    for (int q = 0; q < SP2; ++q)
      S2[q] = make_float2(c_hi + (c_lo + (excl + p[2 * q])), c_hi + (c_lo + (excl + p[2 * q + 1])));
    const float S_first = __shfl_sync(kFullMask, S2[0].x, 0);
    {  // two-sum: c_hi + tot = hi + err exactly
      const float tot = __shfl_sync(kFullMask, incl, 31);
      const float hi = c_hi + tot;
      const float bt = hi - c_hi;
      const float err = (c_hi - (hi - bt)) + (tot - bt);
      c_hi = hi;
      c_lo += err;
    }
    // S_first is the block's smallest sum: a position dead now stays dead
    while (live > 0 && S_first > sh_sd[warp][live - 1]) --live;
    if (live == 0) break;
    float2 pos[SP2], neg[SP2];
#pragma unroll
    for (int q = 0; q < SP2; ++q) pos[q] = neg[q] = make_float2(0.f, 0.f);
    // staged C: the sign of h_in is flipped into C's bits as it is loaded
    constexpr bool XOR = tma && FS::STAGE_C;
#pragma unroll 4
    for (int i = 0; i < live; ++i) {
      const float4 pr = sh_p[warp][i];
      const int2 nq = sh_nq[warp][i];
      float2 cv[SP2];
#pragma unroll
      for (int q = 0; q < SP4; ++q) {
        float4 c4;
        if constexpr (tma && FS::STAGE_C) {
          c4 = fix_lds4x<Tin>(cur + nq.x * FS::ROW + (SP * lane + 4 * q) * FS::ES, (uint32_t)nq.y);
        } else {
          c4 = fix_load4(Cb + (int64_t)nq.x * L, t + 4 * q, t_end, (b * N + nq.x) * L, a.batch * N * L);
        }
        cv[2 * q] = make_float2(c4.x, c4.y);
        cv[2 * q + 1] = make_float2(c4.z, c4.w);
      }
      float2 e[SP2];
#pragma unroll
      for (int q = 0; q < SP2; ++q) {
        const float2 x = __ffma2_rn(S2[q], make_float2(pr.x, pr.y), make_float2(pr.z, pr.w));
        e[q] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      }
      if (XOR) {  // the sign is in cv
#pragma unroll
        for (int q = 0; q < SP2; ++q) pos[q] = __ffma2_rn(cv[q], e[q], pos[q]);
      } else if (nq.y) {  // warp-uniform
#pragma unroll
        for (int q = 0; q < SP2; ++q) neg[q] = __ffma2_rn(cv[q], e[q], neg[q]);
      } else {
#pragma unroll
        for (int q = 0; q < SP2; ++q) pos[q] = __ffma2_rn(cv[q], e[q], pos[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < SP4; ++q) {
      const int64_t tq = t + 4 * q;
      const float2 c01 = __fadd2_rn(pos[2 * q], make_float2(-neg[2 * q].x, -neg[2 * q].y));
      const float2 c23 = __fadd2_rn(pos[2 * q + 1], make_float2(-neg[2 * q + 1].x, -neg[2 * q + 1].y));
      const float4 y4 = tma ? fix_lds4<float>(cur + FS::Y_OFF + 4 * (SP * lane + 4 * q))
                            : fix_load4(yrow, tq, t_end, bd * L, n_act);
      float2 g01 = make_float2(1.f, 1.f), g23 = g01;
      if (zrow) {
        const float4 z4 = tma ? fix_lds4<Tin>(cur + FS::Z_OFF + (SP * lane + 4 * q) * FS::ES)
                              : fix_load4(zrow, tq, t_end, bd * L, n_act);
        g01 = silu_fast2(make_float2(z4.x, z4.y));
        g23 = silu_fast2(make_float2(z4.z, z4.w));
      }
      const float2 o01 = __ffma2_rn(c01, g01, make_float2(y4.x, y4.y));
      const float2 o23 = __ffma2_rn(c23, g23, make_float2(y4.z, y4.w));
      if (tma && tq + 3 < t_end) {
        if (in_range(bd * L + tq, 4, n_act))
          *reinterpret_cast<float4*>(yrow + tq) = make_float4(o01.x, o01.y, o23.x, o23.y);
      } else {
        const float out[4] = {o01.x, o01.y, o23.x, o23.y};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          if (tq + kk < t_end && in_range(bd * L + tq + kk, n_act)) yrow[tq + kk] = out[kk];
      }
    }
    __syncwarp();  // every lane is done with this stage before TMA refills it
    if (tma && k + 2 < nblk) issue(k + 2);
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
