// scan_bwd.cuh -- backward of the selective scan with recomputation.
//
// The forward keeps no states ("Mamba 深度解读报告", sec. 3.3; "Mamba 选择性机制",
// sec. 3.4: the backward recomputes them from the inputs instead of storing
// them).  One CTA owns CH channels of one batch row and the whole sequence:
//
//  pass 1  forward over the sequence, writing only the state at the start of
//          every chunk of T steps to the caller's workspace (skipped when the
//          training forward has written these checkpoints);
//  pass 2  over the chunks in reverse: recompute the chunk's states h_t from
//          its checkpoint into shared memory, then run the adjoint
//          g_t = dq_t C_t + a_{t+1} g_{t+1} backwards through the chunk with
//          the carry in registers:
//            dDelta_t = sum_n g_t (B_t u_t + A a_t h_{t-1}),
//            du_t     = dq_t D + sum_n g_t Delta_t B_t,
//            dA      += g_t Delta_t a_t h_{t-1},
//            dB_t    += g_t Delta_t u_t   (over channels),
//            dC_t    += dq_t h_t          (over channels),
//          with dq_t = dy_t SiLU(z_t), dz_t = dy_t q_t SiLU'(z_t),
//          q_t = C_t . h_t + D u_t, ddelta = dDelta softplus'(x).
//
// Lane layout: G states of one channel per lane (N/G lanes per channel; G = 4
// unless a tuning build sets 2).  Per-channel sums over the states meet by
// xor shuffles among a channel's lanes; sums over the CTA's channels (dB, dC)
// are reduced in shared memory (four states per 16-byte load) and added to HBM
// with one atomic per (state, step) per CTA; dA, dD and the bias gradient
// with one atomic per channel state per CTA.  Those outputs are zeroed by
// the host before the launch.
#pragma once

#include "pointwise.cuh"

namespace ssscan {

struct BwdArgs {
  const void* u;
  const void* delta;
  const void* z;  // nullable
  const void* B;
  const void* C;
  const float* A;
  const float* D;           // nullable
  const float* delta_bias;  // nullable
  const float* dy;          // [batch, dim, L] fp32
  const float* dlast;       // [batch, dim, N] fp32, nullable
  float* du;                // [batch, dim, L]
  float* ddelta;            // [batch, dim, L]
  float* dz;                // [batch, dim, L], nullable (when z is)
  float* dA;                // [dim, N], accumulated
  float* dB;                // [batch, N, L], accumulated
  float* dC;                // [batch, N, L], accumulated
  float* dD;                // [dim], accumulated, nullable
  float* dbias;             // [dim], accumulated, nullable
  float* ckpt;              // [batch][chunks][dim][N]: state at each 16-step chunk start
  int ckpt_given;           // 1: written by the training forward (pass 1 is skipped)
  int64_t batch, dim, seqlen;
  int softplus;
};

template <typename Tin, int N_, int G_ = 4>
struct BwdCfg {
  using Elem = Tin;
  static constexpr int N = N_;
  static constexpr int G = G_;            // states per lane (2 or 4)
  static constexpr int HP = G / 2;        // packed pairs per lane
  static constexpr int K = N / G;         // lanes per channel
  static constexpr int CPW = 32 / K;      // channels per warp
  static constexpr int NWARPS = 4;
  static constexpr int NT = NWARPS * 32;
  static constexpr int CH = NWARPS * CPW; // channels per CTA
  static constexpr int CHP = CH + 1;      // padded row of per-channel values
  static constexpr int T = 16;            // steps per chunk
  static constexpr int ITEMS = CH * T;    // (step, channel) items per chunk
  static constexpr int IPT = (ITEMS + NT - 1) / NT;
  static constexpr int STEP_FLOATS = CH * N;  // one step's states of the CTA
  // row pitch of the per-step states: 16 bytes of padding, so that the
  // 16-byte reads of eight consecutive steps by a quarter-warp in the channel
  // reductions fall on distinct banks
  static constexpr int HB_STRIDE = STEP_FLOATS + 4;
  // staged inputs per thread (register prefetch of the next chunk)
  static constexpr int ACT_PT = (CH * T + NT - 1) / NT;
  static constexpr int SEL_PT = (N * T + NT - 1) / NT;
  // shared memory (floats); per-channel values are [T][CHP] (step-major, so
  // the lanes of a warp read consecutive channels), B and C are [T][N]
  static constexpr int OFF_U = 0;
  static constexpr int OFF_DL = OFF_U + T * CHP;        // delta, then Delta
  static constexpr int OFF_Z = OFF_DL + T * CHP;
  static constexpr int OFF_DY = OFF_Z + T * CHP;        // dy, then dq
  static constexpr int OFF_W = OFF_DY + T * CHP;        // Delta u
  static constexpr int OFF_SG = OFF_W + T * CHP;        // softplus'(x)
  static constexpr int OFF_P1 = OFF_SG + T * CHP;       // per-channel sums (readout, dDelta)
  static constexpr int OFF_P2 = OFF_P1 + T * CHP;       // per-channel sums (du)
  static constexpr int NP = N + 4;                      // B, C row pitch (16-byte aligned)
  // bf16 inputs with four states per lane: B and C stay bf16, a step's row
  // holding 16-byte units [B_4j, B_4j+1, C_4j, C_4j+1, B_4j+2, B_4j+3, C_4j+2,
  // C_4j+3], so that a lane reads its states' B and C in one 16-byte load
  static constexpr bool BC16 = sizeof(Tin) == 2 && G == 4;
  static constexpr int OFF_B = (OFF_P2 + T * CHP + 3) / 4 * 4;  // [T][NP] (BC16: the units)
  static constexpr int OFF_C = OFF_B + T * NP;                  // [T][NP] (not with BC16)
  static constexpr int OFF_H = OFF_C + (BC16 ? 0 : T * NP);     // [T][CH*N] states, then g Delta u
  static constexpr int SMEM_FLOATS = OFF_H + T * HB_STRIDE;
  static constexpr int SMEM_BYTES = SMEM_FLOATS * 4;
  static_assert(N % G == 0 && 32 % K == 0 && (G == 2 || G == 4), "lane split");
  static_assert(ITEMS % NT == 0 || ITEMS < NT, "whole items per thread");
  static constexpr bool ITEM_GUARD = ITEMS < NT;  // some threads have no item
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <typename E>
__device__ __forceinline__ float ld_elem(const E* p, int64_t i) {
  return to_f32(p[i]);
}

__device__ __forceinline__ float sigmoid_fast(float x) {
  return rcp_approx(1.f + ex2_approx(-x * 1.4426950408889634f));
}

// One chunk's inputs in registers (global loads issued early, stored to
// shared memory once the previous chunk is done with it).  Activations are
// read along t (coalesced): element r of a thread is (c, t) = (i / T, i % T),
// i = tid + r * NT.
template <class CF>
struct BwdStage {
  float u[CF::ACT_PT], dl[CF::ACT_PT], z[CF::ACT_PT], dy[CF::ACT_PT];
  float b[CF::SEL_PT], c[CF::SEL_PT];
};

// A thread's fixed element slots: staging slot r is activation element
// (c, t) = (i / T, i % T) and B/C element (n, t) of every chunk, i = tid + r NT;
// item slot it is (c, t) = (i / T, i % T), steps fastest, so that a warp's
// stores of du, ddelta and dz are runs along t.  Their row offsets, validity
// and per-channel constants are computed once, so a chunk only adds t0.
template <class CF>
struct BwdSlots {
  // staging slot r covers element (c, t) = (c0 + r NT/T, t_s) and B/C element
  // (n0 + r NT/T, t_s): offsets are a base plus r times a row stride
  int64_t act0, sel0, row;  // row = (NT / T) L
  int c0, n0, t_s;
  float act_bias[CF::ACT_PT];  // delta_bias of staging slot r's channel
  int64_t item[CF::IPT];    // (b dim + d) L + t of item slot it, or -1 (and its D)
  float D[CF::IPT];
};

template <class CF>
__device__ __forceinline__ void bwd_slots(const BwdArgs& a, int64_t b, int64_t d0,
                                          BwdSlots<CF>& sl) {
  static_assert(CF::NT % CF::T == 0, "staging slots advance by whole rows");
  const int64_t L = a.seqlen;
  sl.c0 = threadIdx.x / CF::T;
  sl.n0 = sl.c0;
  sl.t_s = threadIdx.x - sl.c0 * CF::T;
  sl.row = (int64_t)(CF::NT / CF::T) * L;
  sl.act0 = (b * a.dim + d0 + sl.c0) * L + sl.t_s;
  sl.sel0 = (b * CF::N + sl.n0) * L + sl.t_s;
#pragma unroll
  for (int r = 0; r < CF::ACT_PT; ++r) {
    const int c = sl.c0 + r * (CF::NT / CF::T);
    const bool ok = c < CF::CH && d0 + c < a.dim;
    sl.act_bias[r] = (ok && a.delta_bias) ? __ldg(a.delta_bias + d0 + c) : 0.f;
  }
#pragma unroll
  for (int it = 0; it < CF::IPT; ++it) {
    const int i = threadIdx.x + it * CF::NT;
    const int c = i / CF::T, tt = i - c * CF::T;
    const int64_t d = d0 + c;
    const bool ok = (!CF::ITEM_GUARD || i < CF::ITEMS) && d < a.dim;
    sl.item[it] = ok ? (b * a.dim + d) * L + tt : -1;
    sl.D[it] = (ok && a.D) ? __ldg(a.D + d) : 0.f;
  }
}

template <class CF, bool with_grad>
__device__ __forceinline__ void bwd_fetch(const BwdArgs& a, BwdStage<CF>& st,
                                          const BwdSlots<CF>& sl, int64_t d0, int64_t t0) {
  using E = typename CF::Elem;
  constexpr int RS = CF::NT / CF::T;  // rows per slot step
  const bool t_in = t0 + sl.t_s < a.seqlen;
#pragma unroll
  for (int r = 0; r < CF::ACT_PT; ++r) {
    const int c = sl.c0 + r * RS;
    const bool in = t_in && c < CF::CH && d0 + c < a.dim;
    const int64_t off = sl.act0 + r * sl.row + t0;
    st.u[r] = in ? ld_elem(static_cast<const E*>(a.u), off) : 0.f;
    st.dl[r] = in ? ld_elem(static_cast<const E*>(a.delta), off) : 0.f;
    if (with_grad) {
      st.z[r] = (in && a.z) ? ld_elem(static_cast<const E*>(a.z), off) : 0.f;
      st.dy[r] = in ? a.dy[off] : 0.f;
    }
  }
#pragma unroll
  for (int r = 0; r < CF::SEL_PT; ++r) {
    const bool in = t_in && sl.n0 + r * RS < CF::N;
    const int64_t off = sl.sel0 + r * sl.row + t0;
    st.b[r] = in ? ld_elem(static_cast<const E*>(a.B), off) : 0.f;
    if (with_grad) st.c[r] = in ? ld_elem(static_cast<const E*>(a.C), off) : 0.f;
  }
}

// Store the staged chunk to shared memory, discretising on the way: the
// thread that holds element (c, t) also forms Delta (0 on padding and beyond
// the channels), Delta u and (with_grad) softplus'(x).
template <class CF, bool with_grad>
__device__ __forceinline__ void bwd_store(const BwdArgs& a, const BwdStage<CF>& st,
                                          const BwdSlots<CF>& sl, float* sm, int64_t d0,
                                          int64_t t0) {
  const bool t_in = t0 + sl.t_s < a.seqlen;
#pragma unroll
  for (int r = 0; r < CF::ACT_PT; ++r) {
    const int i = threadIdx.x + r * CF::NT;
    if (i >= CF::CH * CF::T) break;
    const int c = i / CF::T, tt = i - c * CF::T;
    const int o = tt * CF::CHP + c;
    const bool in = t_in && d0 + c < a.dim;
    const float x = st.dl[r] + sl.act_bias[r];
    const float dl = in ? (a.softplus ? softplus_fast(x) : x) : 0.f;
    sm[CF::OFF_U + o] = st.u[r];
    sm[CF::OFF_DL + o] = dl;
    sm[CF::OFF_W + o] = dl * st.u[r];
    if (with_grad) {
      sm[CF::OFF_SG + o] = a.softplus ? sigmoid_fast(x) : 1.f;
      sm[CF::OFF_Z + o] = st.z[r];
      sm[CF::OFF_DY + o] = st.dy[r];
    }
  }
#pragma unroll
  for (int r = 0; r < CF::SEL_PT; ++r) {
    const int i = threadIdx.x + r * CF::NT;
    if (i >= CF::N * CF::T) break;
    const int n = i / CF::T, tt = i - n * CF::T;
    if constexpr (CF::BC16) {  // the values are bf16, so their fp32 high halves are exact
      uint16_t* row = reinterpret_cast<uint16_t*>(sm + CF::OFF_B + tt * CF::NP);
      const int e = 8 * (n >> 2) + 4 * ((n >> 1) & 1) + (n & 1);  // B's place in its unit
      row[e] = (uint16_t)(__float_as_uint(st.b[r]) >> 16);
      if (with_grad) row[e + 2] = (uint16_t)(__float_as_uint(st.c[r]) >> 16);
    } else {
      sm[CF::OFF_B + tt * CF::NP + n] = st.b[r];
      if (with_grad) sm[CF::OFF_C + tt * CF::NP + n] = st.c[r];
    }
  }
}

// Sum over the K lanes of a channel (consecutive lanes of one warp).
template <int K>
__device__ __forceinline__ float lane_sum(float v) {
#pragma unroll
  for (int off = K / 2; off > 0; off >>= 1) v += __shfl_xor_sync(kFullMask, v, off);
  return v;
}

template <class CF>
__global__ void __launch_bounds__(CF::NT)
    scan_bwd_kernel(const BwdArgs a) {
  constexpr int N = CF::N, G = CF::G, K = CF::K, T = CF::T, CHP = CF::CHP;
  extern __shared__ __align__(16) float sm[];
  const int64_t tiles = (a.dim + CF::CH - 1) / CF::CH;
  const int64_t b = blockIdx.x / tiles;
  const int64_t d0 = (blockIdx.x - b * tiles) * CF::CH;
  const int64_t L = a.seqlen;
  const int64_t nk = (L + T - 1) / T;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = warp * CF::CPW + lane / K;  // this lane's channel
  const int j = lane % K;                   // its state group
  const int64_t d = d0 + c;
  const bool chan_ok = d < a.dim;
  // this lane's states in checkpoint k: ckpt[b][k][d][j G ..]
  const int64_t ck_stride = a.dim * N;
  float* ck_lane = a.ckpt + (b * nk * a.dim + d) * N + j * G;
  float* hb = sm + CF::OFF_H;

  constexpr int HP = CF::HP;
  // decay constants of this lane's G states, as HP packed pairs
  float2 A2[HP], An[HP];
#pragma unroll
  for (int p = 0; p < HP; ++p) {
    const float a0 = chan_ok ? __ldg(a.A + d * N + j * G + 2 * p) : 0.f;
    const float a1 = chan_ok ? __ldg(a.A + d * N + j * G + 2 * p + 1) : 0.f;
    An[p] = make_float2(a0, a1);
    A2[p] = make_float2(a0 * 1.4426950408889634f, a1 * 1.4426950408889634f);
  }
  BwdStage<CF> st;
  BwdSlots<CF> sl;
  bwd_slots<CF>(a, b, d0, sl);
  auto ex2_pair = [](float2 x) { return make_float2(ex2_approx(x.x), ex2_approx(x.y)); };
  auto ld_pairs = [](const float* p, float2 (&v)[HP]) {  // one 16- or 8-byte load
    if constexpr (HP == 2) {
      const float4 q = *reinterpret_cast<const float4*>(p);
      v[0] = make_float2(q.x, q.y);
      v[HP - 1] = make_float2(q.z, q.w);
    } else {
      v[0] = *reinterpret_cast<const float2*>(p);
    }
  };
  auto st_pairs = [](float* p, const float2 (&v)[HP]) {
    if constexpr (HP == 2)
      *reinterpret_cast<float4*>(p) = make_float4(v[0].x, v[0].y, v[HP - 1].x, v[HP - 1].y);
    else
      *reinterpret_cast<float2*>(p) = v[0];
  };
  // B (and C) of this lane's states at step t of the staged chunk
  auto ld_bc = [&](int t, float2 (&bb)[HP], float2 (&cc)[HP]) {
    if constexpr (CF::BC16) {
      const uint4 v = *reinterpret_cast<const uint4*>(sm + CF::OFF_B + t * CF::NP + j * G);
      auto lo = [](uint32_t x) { return __uint_as_float(x << 16); };
      auto hi = [](uint32_t x) { return __uint_as_float(x & 0xffff0000u); };
      bb[0] = make_float2(lo(v.x), hi(v.x));
      cc[0] = make_float2(lo(v.y), hi(v.y));
      bb[HP - 1] = make_float2(lo(v.z), hi(v.z));
      cc[HP - 1] = make_float2(lo(v.w), hi(v.w));
    } else {
      ld_pairs(sm + CF::OFF_B + t * CF::NP + j * G, bb);
      ld_pairs(sm + CF::OFF_C + t * CF::NP + j * G, cc);
    }
  };
  auto ld_b = [&](int t, float2 (&bb)[HP]) {
    if constexpr (CF::BC16) {
      float2 cc[HP];
      ld_bc(t, bb, cc);
    } else {
      ld_pairs(sm + CF::OFF_B + t * CF::NP + j * G, bb);
    }
  };
  auto zero_pairs = [](float2 (&v)[HP]) {
#pragma unroll
    for (int p = 0; p < HP; ++p) v[p] = make_float2(0.f, 0.f);
  };
  float* hb_lane = hb + c * N + j * G;        // and in every step row of hb

  // ---- pass 1: forward, checkpoint the state at every chunk start ----
  // (skipped when the training forward has written the checkpoints)
  float2 h[HP];
  zero_pairs(h);
  if (!a.ckpt_given) bwd_fetch<CF, false>(a, st, sl, d0, 0);
  for (int64_t k = 0; k < nk && !a.ckpt_given; ++k) {
    if (chan_ok) st_pairs(ck_lane + k * ck_stride, h);
    bwd_store<CF, false>(a, st, sl, sm, d0, k * T);
    if (k + 1 < nk) bwd_fetch<CF, false>(a, st, sl, d0, (k + 1) * T);
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < T; ++t) {
      const float dl = sm[CF::OFF_DL + t * CHP + c], w = sm[CF::OFF_W + t * CHP + c];
      const float2 dl2 = make_float2(dl, dl), w2 = make_float2(w, w);
      float2 bb[HP];
      ld_b(t, bb);
#pragma unroll
      for (int p = 0; p < HP; ++p)
        h[p] = __ffma2_rn(ex2_pair(__fmul2_rn(dl2, A2[p])), h[p], __fmul2_rn(w2, bb[p]));
    }
    __syncthreads();
  }

  // ---- pass 2: chunks in reverse ----
  float2 carry[HP];
#pragma unroll
  for (int p = 0; p < HP; ++p) {
    const float* dl_ = a.dlast + (b * a.dim + d) * N + j * G + 2 * p;
    carry[p] = (a.dlast && chan_ok) ? make_float2(dl_[0], dl_[1]) : make_float2(0.f, 0.f);
  }
  float2 dA_acc[HP];
  zero_pairs(dA_acc);
  float dD_acc[CF::IPT], db_acc[CF::IPT];
#pragma unroll
  for (int it = 0; it < CF::IPT; ++it) dD_acc[it] = db_acc[it] = 0.f;

  bwd_fetch<CF, true>(a, st, sl, d0, (nk - 1) * T);
  float2 ck_next[HP];
  zero_pairs(ck_next);
  // the checkpoint of the chunk to come, loaded a chunk early (the same thread
  // wrote it in pass 1, or the training forward did before this launch)
  if (chan_ok) ld_pairs(ck_lane + (nk - 1) * ck_stride, ck_next);
  for (int64_t k = nk - 1; k >= 0; --k) {
    const int64_t t0 = k * T;
    float2 h_start[HP];
#pragma unroll
    for (int p = 0; p < HP; ++p) h_start[p] = ck_next[p];
    bwd_store<CF, true>(a, st, sl, sm, d0, t0);
    if (k > 0) {
      bwd_fetch<CF, true>(a, st, sl, d0, (k - 1) * T);
      if (chan_ok) ld_pairs(ck_lane + (k - 1) * ck_stride, ck_next);
    }
    __syncthreads();
    // recompute the chunk's states from its checkpoint; channel readouts
    float2 hs[HP];
#pragma unroll
    for (int p = 0; p < HP; ++p) hs[p] = h_start[p];
#pragma unroll 4
    for (int t = 0; t < T; ++t) {
      const float dl = sm[CF::OFF_DL + t * CHP + c], w = sm[CF::OFF_W + t * CHP + c];
      const float2 dl2 = make_float2(dl, dl), w2 = make_float2(w, w);
      float2 bb[HP], cc[HP];
      ld_bc(t, bb, cc);
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int p = 0; p < HP; ++p) {
        hs[p] = __ffma2_rn(ex2_pair(__fmul2_rn(dl2, A2[p])), hs[p], __fmul2_rn(w2, bb[p]));
        acc = __ffma2_rn(cc[p], hs[p], acc);
      }
      st_pairs(hb_lane + t * CF::HB_STRIDE, hs);
      const float part = lane_sum<K>(acc.x + acc.y);
      if (j == 0) sm[CF::OFF_P1 + t * CHP + c] = part;
    }
    __syncthreads();
    // per item: q, the gate's derivatives, dq
#pragma unroll
    for (int it = 0; it < CF::IPT; ++it) {
      const int i = tid + it * CF::NT;
      if (CF::ITEM_GUARD && i >= CF::ITEMS) break;
      const int ci = i / CF::T, tt = i - ci * CF::T;
      const int o = tt * CHP + ci;
      const bool in = sl.item[it] >= 0 && t0 + tt < L;
      const float uu = sm[CF::OFF_U + o];
      const float q = sm[CF::OFF_P1 + o] + sl.D[it] * uu;
      const float dy = sm[CF::OFF_DY + o];
      float dq = dy;
      if (a.z) {
        const float zz = sm[CF::OFF_Z + o];
        const float sg = sigmoid_fast(zz);
        dq = dy * zz * sg;
        if (in) a.dz[sl.item[it] + t0] = dy * q * sg * (1.f + zz * (1.f - sg));
      }
      sm[CF::OFF_DY + o] = dq;
      if (in) dD_acc[it] = fmaf(dq, uu, dD_acc[it]);
    }
    __syncthreads();
    // dC[b, n, t] += sum_c dq[t, c] h_t[c, n], four consecutive states per
    // item, steps fastest (a warp's atomics are runs along t)
    for (int i = tid; i < (N / 4) * T; i += CF::NT) {
      const int n = 4 * (i / T), tt = i - (n / 4) * T;
      if (t0 + tt >= L) continue;
      float2 s01 = make_float2(0.f, 0.f), s23 = s01;
      const float* hr = hb + tt * CF::HB_STRIDE + n;
#pragma unroll 8
      for (int cc = 0; cc < CF::CH; ++cc) {
        const float dq = sm[CF::OFF_DY + tt * CHP + cc];
        const float4 h4 = *reinterpret_cast<const float4*>(hr + cc * N);
        s01 = __ffma2_rn(make_float2(dq, dq), make_float2(h4.x, h4.y), s01);
        s23 = __ffma2_rn(make_float2(dq, dq), make_float2(h4.z, h4.w), s23);
      }
      float* dst = a.dC + (b * N + n) * L + t0 + tt;
      atomicAdd(dst, s01.x);
      atomicAdd(dst + L, s01.y);
      atomicAdd(dst + 2 * L, s23.x);
      atomicAdd(dst + 3 * L, s23.y);
    }
    __syncthreads();
    // the adjoint, backwards through the chunk
#pragma unroll 2
    for (int t = T - 1; t >= 0; --t) {
      const float dl = sm[CF::OFF_DL + t * CHP + c];
      const float uu = sm[CF::OFF_U + t * CHP + c];
      const float dq = sm[CF::OFF_DY + t * CHP + c];
      const float w = sm[CF::OFF_W + t * CHP + c];
      const float2 dl2 = make_float2(dl, dl), w2 = make_float2(w, w), dq2 = make_float2(dq, dq);
      float2 bb[HP], cc[HP], prev[HP];
      ld_bc(t, bb, cc);
      if (t > 0) {
        ld_pairs(hb_lane + (t - 1) * CF::HB_STRIDE, prev);
      } else {
#pragma unroll
        for (int p = 0; p < HP; ++p) prev[p] = h_start[p];
      }
      // per state: g_t, and with a_t h_{t-1} (eprev) the terms of
      //   dDelta_t = u_t sum_n g B + sum_n g A a h_{t-1},  du_t - dq D = Delta_t sum_n g B,
      //   dA += Delta_t g a h_{t-1},  dB_t += g Delta_t u_t
      float2 gB = make_float2(0.f, 0.f), gAe = make_float2(0.f, 0.f), gdu[HP];
#pragma unroll
      for (int p = 0; p < HP; ++p) {
        const float2 e = ex2_pair(__fmul2_rn(dl2, A2[p]));
        const float2 gt = __ffma2_rn(dq2, cc[p], carry[p]);
        const float2 ge = __fmul2_rn(gt, __fmul2_rn(e, prev[p]));
        gB = __ffma2_rn(gt, bb[p], gB);
        gAe = __ffma2_rn(An[p], ge, gAe);
        dA_acc[p] = __ffma2_rn(dl2, ge, dA_acc[p]);
        gdu[p] = __fmul2_rn(gt, w2);
        carry[p] = __fmul2_rn(e, gt);
      }
      // h_t is no longer needed (its dC and its step's prev are done): reuse the slot
      st_pairs(hb_lane + t * CF::HB_STRIDE, gdu);
      const float gB_c = lane_sum<K>(gB.x + gB.y);
      const float gAe_c = lane_sum<K>(gAe.x + gAe.y);
      if (j == 0) {
        sm[CF::OFF_P1 + t * CHP + c] = fmaf(uu, gB_c, gAe_c);
        sm[CF::OFF_P2 + t * CHP + c] = dl * gB_c;
      }
    }
    __syncthreads();
    // dB[b, n, t] += sum_c g Delta u, four consecutive states per item, steps fastest
    for (int i = tid; i < (N / 4) * T; i += CF::NT) {
      const int n = 4 * (i / T), tt = i - (n / 4) * T;
      if (t0 + tt >= L) continue;
      float2 s01 = make_float2(0.f, 0.f), s23 = s01;
      const float* hr = hb + tt * CF::HB_STRIDE + n;
#pragma unroll 8
      for (int cc = 0; cc < CF::CH; ++cc) {
        const float4 g4 = *reinterpret_cast<const float4*>(hr + cc * N);
        s01 = __fadd2_rn(s01, make_float2(g4.x, g4.y));
        s23 = __fadd2_rn(s23, make_float2(g4.z, g4.w));
      }
      float* dst = a.dB + (b * N + n) * L + t0 + tt;
      atomicAdd(dst, s01.x);
      atomicAdd(dst + L, s01.y);
      atomicAdd(dst + 2 * L, s23.x);
      atomicAdd(dst + 3 * L, s23.y);
    }
    // per item: du, ddelta, the bias gradient
#pragma unroll
    for (int it = 0; it < CF::IPT; ++it) {
      const int i = tid + it * CF::NT;
      if (CF::ITEM_GUARD && i >= CF::ITEMS) break;
      const int ci = i / CF::T, tt = i - ci * CF::T;
      const int o = tt * CHP + ci;
      if (sl.item[it] < 0 || t0 + tt >= L) continue;
      const float dx = sm[CF::OFF_P1 + o] * sm[CF::OFF_SG + o];
      const int64_t off = sl.item[it] + t0;
      a.ddelta[off] = dx;
      a.du[off] = fmaf(sm[CF::OFF_DY + o], sl.D[it], sm[CF::OFF_P2 + o]);
      db_acc[it] += dx;
    }
    __syncthreads();
  }

  // per-channel sums over this CTA's part of the batch
  if (chan_ok) {
#pragma unroll
    for (int p = 0; p < HP; ++p) {
      atomicAdd(a.dA + d * N + j * G + 2 * p, dA_acc[p].x);
      atomicAdd(a.dA + d * N + j * G + 2 * p + 1, dA_acc[p].y);
    }
  }
#pragma unroll
  for (int it = 0; it < CF::IPT; ++it) {
    const int i = tid + it * CF::NT;
    if (CF::ITEM_GUARD && i >= CF::ITEMS) break;
    const int64_t di = d0 + i / CF::T;
    if (di >= a.dim) continue;
    if (a.dD) atomicAdd(a.dD + di, dD_acc[it]);
    if (a.dbias) atomicAdd(a.dbias + di, db_acc[it]);
  }
}

}  // namespace ssscan
