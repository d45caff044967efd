// scan_fwd_chunked.cuh -- channel-parallel fused selective-scan forward.
//
// One CTA owns CH consecutive channels d of one batch row b and walks the
// whole sequence in chunks of T timesteps.  Inside the CTA a warp holds
// 32/K channels; the K lanes of a channel each keep G = N/K of its states
// h[n] in fp32 registers for the whole sequence, so the state never touches
// memory (the SRAM-resident scan of "Mamba 深度解读报告", sec. 2.4, and the
// fused discretise/scan/readout kernel of "Mamba 选择性机制", sec. 3.2).
//
// Per chunk, with the inputs staged in shared memory (TMA tiles, double
// buffered on mbarriers, so the next chunk's copy overlaps this chunk's math):
//   phase 1  per element: Delta = softplus(delta + bias), w = Delta * u, kept
//            as float4 of four timesteps; B_t and C_t transposed from their
//            [n][t] rows into 16-byte units per step [B_2p, B_2p+1, C_2p,
//            C_2p+1, ...] in the input dtype (four bf16 or two fp32 states a
//            unit), a lane's units interleaved with its neighbours' so that a
//            quarter-warp reads 128 contiguous bytes;
//   phase 2  per (channel, state): A_bar = 2^(Delta * A * log2 e),
//            h = A_bar * h + w * B_t[n], and the lane's partial readout
//            sum_n C_t[n] h[n], in packed fp32x2 arithmetic; B_t and C_t are
//            staged once per CTA and read by every channel (the per-token
//            sharing of "从Transformer的痛点 ... Mamba", sec. 4.2);
//   phase 3  per element: s = sum of the K lane partials,
//            y = (s + D u) * SiLU(z), coalesced fp32 stores.
// The serial time loop inside a thread is the recurrence itself.  Where a
// time range starts with its carry-in unknown, the associative operator of
// "Mamba 选择性机制", sec. 3.1, joins it to what came before: the time-split
// warps of a CTA (phase2_split, short sequences over few channels), the
// balanced schedule's carries between CTAs, and the segments of a long
// sequence scanned at once from h = 0, whose end states and sums of Delta the
// correction kernel (scan_fix.cuh) folds into each segment's carry-in.
//
// With two channels per lane (CPL = 2) a lane keeps the same G states of two
// channels and packs its fp32x2 arithmetic over the channel pair: the pair's
// Delta and w arrive together from shared memory, and every B_t[n], C_t[n] a
// lane widens serves both channels (half the shared-memory traffic and
// conversions per state of the one-channel layout).
//
// Shared-memory layouts are chosen so that each quarter-warp (the unit a
// 16-byte access is serviced in) touches distinct banks.  Rows whose start
// is not 16-byte aligned (odd L, offset views) take an element-wise load
// path instead of TMA.
#pragma once

#include <cuda.h>

#include "pointwise.cuh"

namespace ssscan {

struct FwdArgs {
  const void* u;
  const void* delta;
  const void* z;  // nullable
  const void* B;
  const void* C;
  const float* A;
  const float* D;           // nullable
  const float* delta_bias;  // nullable
  float* y;
  float* last_state;  // nullable
  const float* h0;    // [batch, dim, N] initial state, nullable (zero); may be last_state
  // fused short convolution (kernels built with CONV): u holds the
  // convolution's input x; conv_w [dim, conv_width <= kConvTaps], conv_b [dim]
  const float* conv_w;
  const float* conv_b;  // nullable
  int conv_width;
  // training checkpoints: the state at the start of every 16-step chunk,
  // [batch][ceil(L / 16)][dim][N] fp32 (nullable: not written)
  float* ckpt;
  // sequence segments (Sched::nseg > 1): the state each segment ends in,
  // scanned from h = 0 (segment 0: from h0), [batch * dim][nseg][N], and the
  // sum of Delta over each segment, [batch * dim][nseg]
  float* seg_h;
  float* seg_dsum;
  int64_t batch, dim, seqlen;
  int softplus;
  int vec;  // 1: TMA path (16-byte aligned rows); 0: element-wise loads
};

// TMA descriptors for the five input tiles ([B][D][L] activations with a
// [1][CH][T] box, [B][N][L] selection parameters with a [1][N][T] box).
struct FwdMaps {
  CUtensorMap u, delta, z, B, C;
};

constexpr uint32_t kTmaSpinLimit = 1u << 24;
constexpr int kConvTaps = 4;  // widest fused convolution

// Where this lane writes training checkpoints for the current chunk: its
// states' slot in the chunk's first 16-step checkpoint (null: none), the
// distance to the next checkpoint, and the steps of the sequence left from
// the chunk start.
struct CkptCtx {
  float* p;
  int64_t stride;
  int64_t left;
};

// Tin: input dtype; N: states per channel; K: lanes per channel (per channel
// pair with CPL = 2); NWARPS: warps per CTA; T: timesteps per chunk; CPL:
// channels per lane (1 or 2).  CONV: the u input is the pre-convolution x,
// staged with HALO earlier steps per row, and phase 1 forms
// u = SiLU(conv(x) + bias).  ZOH: exact zero-order-hold B_bar.  TRAIN: the
// state at every 16-step chunk start is written out for the backward.  The
// variants (CONV, ZOH, TRAIN) use one channel per lane.  WT: warps that split
// each chunk in time (1: every warp walks the whole chunk for its own
// channels; > 1, one channel per lane only: WT warps share one set of
// channels, each scanning T/WT consecutive steps of the chunk, joined with the
// associative operator; for short sequences over few channels).
template <typename Tin, int N_, int K_, int NWARPS_, int T_, int CPL_ = 1, bool CONV_ = false,
          bool ZOH_ = false, bool TRAIN_ = false, int WT_ = 1>
struct ChunkedCfg {
  using Elem = Tin;
  static constexpr int N = N_;            // states per channel
  static constexpr int K = K_;            // lanes per channel (or channel pair)
  static constexpr int G = N / K;         // states per lane and channel
  static constexpr int CPL = CPL_;        // channels per lane
  static constexpr int HP = CPL == 1 ? G / 2 : G;  // float2 registers per lane state
  static constexpr int NWARPS = NWARPS_;
  static constexpr int T = T_;            // timesteps per chunk
  static constexpr int WT = WT_;          // time-split warps per channel set
  static constexpr int WC = NWARPS / WT;  // warps across channels
  static constexpr int TW = T / WT;       // steps per warp per chunk
  static constexpr int LGW = 32 / K;      // lane groups per warp
  static constexpr int LG = WC * LGW;     // lane groups per CTA
  static constexpr int CH = LG * CPL;     // channels per CTA
  static constexpr int NT = NWARPS * 32;
  static constexpr int ES = (int)sizeof(Tin);
  static constexpr int QPR = T / 4;                  // 4-step quads per row
  static constexpr bool CONV = CONV_;
  static constexpr bool ZOH = ZOH_;
  static constexpr bool TRAIN = TRAIN_;
  // x steps staged before the chunk: >= kConvTaps - 1, and a whole number of
  // 16-byte units so that the shifted TMA box stays aligned
  static constexpr int HALO = CONV ? 8 : 0;
  static constexpr int XT = T + HALO;                // u (or x) row length
  static constexpr int ACT_TILE = CH * T * ES;       // one delta or z tile (bytes)
  static constexpr int X_TILE = CH * XT * ES;        // the u (or x) tile (bytes)
  static constexpr int SEL_TILE = N * T * ES;        // one B or C tile (bytes)
  // raw stage: [u or x: CH rows of XT][delta: CH x T][z: CH x T][B: N x T][C: N x T]
  static constexpr int OFF_DELTA_T = X_TILE;
  static constexpr int OFF_Z_T = X_TILE + ACT_TILE;
  static constexpr int OFF_B_T = X_TILE + 2 * ACT_TILE;
  static constexpr int OFF_C_T = OFF_B_T + SEL_TILE;
  static constexpr int RAW_BYTES = OFF_C_T + SEL_TILE;
  // Delta and w per (quad, channel) as float4 of four steps; with CPL = 2 a
  // lane group's two float4 hold its channel pair interleaved by step:
  // {c0 t0, c1 t0, c0 t1, c1 t1}, {c0 t2, c1 t2, c0 t3, c1 t3}.  The row pitch
  // (float4 units) is odd, so a quarter-warp's writes hit distinct banks.
  static constexpr int DW_STRIDE = CH + 1;
  static constexpr int DW_BYTES = QPR * DW_STRIDE * 16;
  static constexpr int BCES = ES;  // bytes of one B or C value in the transposed tile
  static constexpr int PAIR_BYTES = 4 * BCES;        // one state pair: B_lo, B_hi, C_lo, C_hi
  static constexpr int BC_BLOCK = 2 * PAIR_BYTES;    // two pairs: four states
  static constexpr int BC_DATA = (N / 4) * BC_BLOCK; // bytes of one timestep
  // A timestep's B, C are 16-byte units (four bf16 states or two fp32
  // states); lane j of a channel owns UPL units.  With more than one unit per
  // lane they are stored unit-major, unit h of lane j at position h K + j, so
  // that the lanes of a quarter-warp load 16 consecutive bytes each (one
  // 128-byte wavefront) rather than every other 16 (two).
  static constexpr int UNIT_STATES = 16 / (2 * BCES);
  static constexpr int UPL = G / UNIT_STATES;         // units per lane (0: half a unit)
  static constexpr bool BC_PERMUTE = UPL >= 2;
  static constexpr int UNIT_STRIDE = BC_PERMUTE ? K * 16 : 16;  // between a lane's units
  __host__ __device__ static constexpr int bc_pos(int u) {  // byte offset of unit u
    return (BC_PERMUTE ? (u % UPL) * K + u / UPL : u) * 16;
  }
  // The bf16 transpose of phase 1 (T = 32) runs its items step-fastest: a
  // quarter-warp writes the same unit of rows 2 tp, tp = 8 consecutive values,
  // so a row pitch of 16 mod 64 bytes spreads those writes over four bank
  // quarters (two-way at most).  The fp32 transpose runs blocks-fastest, and a
  // pitch of 32 mod 64 puts its rows 2tp and 2tp+2 on opposite bank halves.
  static constexpr bool TP_FAST = ES == 2 && T == 32;
  static constexpr int BC_ROW = TP_FAST ? (BC_DATA % 64 == 0 ? BC_DATA + 16 : BC_DATA)
                                        : ((BC_DATA % 128 == 64) ? BC_DATA + 32 : BC_DATA);
  static constexpr int BC_BYTES = T * BC_ROW;
  static constexpr int SY_STRIDE = T + 4;            // floats per (channel, lane) row
  static constexpr int SY_BYTES = CH * K * SY_STRIDE * 4;
  static constexpr int OFF_RAW1 = RAW_BYTES;
  static constexpr int OFF_DWD = 2 * RAW_BYTES;
  static constexpr int OFF_DWW = OFF_DWD + DW_BYTES;
  static constexpr int OFF_BC = OFF_DWW + DW_BYTES;
  static constexpr int OFF_SY = OFF_BC + BC_BYTES;
  // time-split aggregates: (prod A_bar, local end state) per warp and lane state
  static constexpr int AGG_FLOATS = WT > 1 ? WT * WC * 32 * G : 0;
  static constexpr int OFF_AGG = OFF_SY + SY_BYTES;
  // CONV: u = SiLU(conv) per (quad, channel), for phase 3's D u
  static constexpr int SU_BYTES = CONV ? DW_BYTES : 0;
  static constexpr int OFF_SU = OFF_AGG + 2 * AGG_FLOATS * 4;
  // ZOH: 1 / Delta per (quad, channel)
  static constexpr int DWI_BYTES = ZOH ? DW_BYTES : 0;
  static constexpr int OFF_DWI = OFF_SU + SU_BYTES;
  static constexpr int SMEM_USED = OFF_DWI + DWI_BYTES;
  static constexpr int SMEM_BYTES = SMEM_USED + 128;  // slack to align the base to 128 bytes
  // CTAs per SM the register budget must allow (shared memory permitting)
  // (at most 512 threads' worth: a 128-register budget per thread)
  static constexpr int SMEM_CTAS = 227 * 1024 / (SMEM_USED + 128 + 1024);
  static constexpr int THREAD_CTAS = 512 / NT > 0 ? 512 / NT : 1;
  static constexpr int MIN_CTAS = SMEM_CTAS < THREAD_CTAS ? SMEM_CTAS : THREAD_CTAS;
  // phase 1 works on (lane group, quad) items (CPL channels x 4 steps each),
  // phase 3 on (channel, quad) items
  static constexpr int ITEMS1 = LG * QPR;
  static constexpr int ITEMS1_PER_THREAD = (ITEMS1 + NT - 1) / NT;
  static constexpr int ITEMS = CH * QPR;
  static constexpr int ITEMS_PER_THREAD = (ITEMS + NT - 1) / NT;

  static_assert(N % K == 0 && 32 % K == 0, "lane split");
  static_assert(CPL == 1 || CPL == 2, "channels per lane");
  static_assert(CPL == 1 || (!CONV && !ZOH && !TRAIN), "the variants use one channel per lane");
  static_assert(NWARPS % WT == 0 && T % (4 * WT) == 0 && (WT == 1 || CPL == 1), "time split");
  static_assert(CPL == 2 || G % 2 == 0, "a lane holds whole state pairs");
  static_assert(G % 4 == 0 || (CPL == 1 && G % 2 == 0), "B, C loads of whole state pairs");
  static_assert(T % 8 == 0 && (T * ES) % 16 == 0 && T <= 256 && CH <= 256, "TMA box");
  static_assert(ACT_TILE % 128 == 0 && SEL_TILE % 128 == 0 && X_TILE % 128 == 0,
                "TMA destinations 128-byte aligned");
  static_assert(!CONV || ((HALO * ES) % 16 == 0 && HALO >= kConvTaps - 1 && XT <= 256),
                "convolution halo");
  static_assert(T % 16 == 0 && (WT == 1 || 16 % TW == 0),
                "16-step checkpoints fall on quad or warp-segment starts");
  static_assert(DW_BYTES % 16 == 0 && BC_BYTES % 16 == 0, "alignment");
  static_assert((ITEMS % NT == 0 || ITEMS < NT) && (ITEMS1 % NT == 0 || ITEMS1 < NT),
                "whole items per thread");
  static_assert(QPR <= 32 && (NT % QPR) == 0, "an item's quads are lanes of one warp");
  static constexpr bool ITEM_GUARD = ITEMS < NT;    // some threads have no phase-3 item
  static constexpr bool ITEM1_GUARD = ITEMS1 < NT;  // some threads have no phase-1 item
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Quads of timesteps the recurrence loop is unrolled by (tuning builds may
// override it).
#ifndef SS_PHASE2_UNROLL
#define SS_PHASE2_UNROLL 2
#endif
constexpr int kPhase2Unroll = SS_PHASE2_UNROLL;

// Both halves of a packed bf16 pair as fp32 (exact).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// ---------------------------------------------------------------- loads ---

template <class CF>
__device__ __forceinline__ uint32_t chunk_tx_bytes(bool has_z) {
  return CF::X_TILE + (has_z ? 2 : 1) * CF::ACT_TILE + 2 * CF::SEL_TILE;
}

// Issue the TMA loads of chunk t0 into one raw stage (one thread).
template <class CF>
__device__ __forceinline__ void tma_chunk(const FwdMaps& m, unsigned char* raw, uint64_t* bar,
                                          int32_t b, int32_t d0, int32_t t0, bool has_z) {
  fence_proxy_async_smem();
  mbar_arrive_expect_tx(bar, chunk_tx_bytes<CF>(has_z));
  // the x box starts HALO steps early (zero fill before t = 0); HALO * size
  // is a multiple of 16 bytes, so the start stays 16-byte aligned
  tma_load_3d(raw, &m.u, bar, t0 - CF::HALO, d0, b);
  tma_load_3d(raw + CF::OFF_DELTA_T, &m.delta, bar, t0, d0, b);
  if (has_z) tma_load_3d(raw + CF::OFF_Z_T, &m.z, bar, t0, d0, b);
  tma_load_3d(raw + CF::OFF_B_T, &m.B, bar, t0, 0, b);
  tma_load_3d(raw + CF::OFF_C_T, &m.C, bar, t0, 0, b);
}

// Element-wise fallback for rows that TMA cannot address (all threads); the
// same stage layout as tma_chunk, zeros outside the tensors.
template <class CF>
__device__ __forceinline__ void load_chunk_scalar(const FwdArgs& a, typename CF::Elem* raw,
                                                  int64_t b, int64_t d0, int64_t t0) {
  using E = typename CF::Elem;
  const int64_t L = a.seqlen;
  // u (or x with its halo): CH rows of XT steps from t0 - HALO
  for (int i = threadIdx.x; i < CF::CH * CF::XT; i += CF::NT) {
    const int c = i / CF::XT, tt = i - c * CF::XT;
    const int64_t t = t0 - CF::HALO + tt, d = d0 + c;
    E val = zero_elem<E>();
    if (t >= 0 && t < L && d < a.dim) {
      const int64_t ix = (b * a.dim + d) * L + t;
      if (in_range(ix, a.batch * a.dim * L)) val = static_cast<const E*>(a.u)[ix];
    }
    raw[i] = val;
  }
  // delta, z, B, C: [2 CH + 2 N] rows of T steps
  E* rest = raw + CF::CH * CF::XT;
  for (int i = threadIdx.x; i < (2 * CF::CH + 2 * CF::N) * CF::T; i += CF::NT) {
    const int r = i / CF::T, tt = i - r * CF::T;
    const int64_t t = t0 + tt;
    E val = zero_elem<E>();
    if (t < L) {
      if (r < 2 * CF::CH) {
        const int which = r / CF::CH, c = r - which * CF::CH;
        const int64_t d = d0 + c;
        const void* base = which == 0 ? a.delta : a.z;
        const int64_t ix = (b * a.dim + d) * L + t;
        if (d < a.dim && base && in_range(ix, a.batch * a.dim * L))
          val = static_cast<const E*>(base)[ix];
      } else {
        const int rr = r - 2 * CF::CH, which = rr / CF::N, n = rr - which * CF::N;
        const int64_t ix = (b * CF::N + n) * L + t;
        if (in_range(ix, a.batch * CF::N * L)) val = static_cast<const E*>(which == 0 ? a.B : a.C)[ix];
      }
    }
    rest[i] = val;
  }
}

// ------------------------------------------------------------- phase 1 ---

// Per (channel, 4-step quad) item, spread over the CTA's threads.  The same
// item-to-thread map is used by phase 3, so a thread's per-channel constants
// (bias, convolution taps, D) stay in its registers.
template <class CF>
struct ConvRegs {  // per-item convolution taps, right-aligned: tap kConvTaps-1 meets step t
  float w[CF::CONV ? CF::ITEMS1_PER_THREAD : 1][kConvTaps];
  float b[CF::CONV ? CF::ITEMS1_PER_THREAD : 1];
};

template <class CF, bool kFull>
__device__ __forceinline__ void phase1(const FwdArgs& a, const typename CF::Elem* raw,
                                       float4* dwD, float4* dwW, float4* dwI, float4* su,
                                       unsigned char* bc,
                                       const float (&bias_it)[CF::ITEMS1_PER_THREAD][CF::CPL],
                                       const ConvRegs<CF>& cv, int64_t d0, int64_t t0,
                                       double (&dsum)[CF::ITEMS1_PER_THREAD][CF::CPL], bool seg) {
  using E = typename CF::Elem;
  const int tid = threadIdx.x;
  const E* rawD = raw + CF::CH * CF::XT;
#pragma unroll
  for (int it = 0; it < CF::ITEMS1_PER_THREAD; ++it) {
    const int i = tid + it * CF::NT;
    if (CF::ITEM1_GUARD && i >= CF::ITEMS1) break;
    const int lg = i / CF::QPR, q = i - lg * CF::QPR;
    float delt[CF::CPL][4], w[CF::CPL][4];
#pragma unroll
    for (int cc = 0; cc < CF::CPL; ++cc) {
      const int c = lg * CF::CPL + cc;
      const float4 dl = load4_f32(rawD + c * CF::T + 4 * q);
      float4 uu;
      if constexpr (CF::CONV) {
        // u = SiLU(b + sum_k w[k] x[t - (kConvTaps-1) + k]); the row holds x from
        // step t0 - HALO, so steps t0+4q-4 .. t0+4q+3 are elements 4q+HALO-4 ..
        const E* xr = raw + c * CF::XT + 4 * q + CF::HALO - 4;
        const float4 xa = load4_f32(xr), xb = load4_f32(xr + 4);
        const float win[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        float o[4];
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          float acc = cv.b[it];
#pragma unroll
          for (int k = 0; k < kConvTaps; ++k) acc = fmaf(cv.w[it][k], win[k4 + 5 - kConvTaps + k], acc);
          o[k4] = acc;
        }
        const float2 u01 = silu_fast2(make_float2(o[0], o[1]));
        const float2 u23 = silu_fast2(make_float2(o[2], o[3]));
        uu = make_float4(u01.x, u01.y, u23.x, u23.y);
        su[q * CF::DW_STRIDE + c] = uu;
      } else {
        uu = load4_f32(raw + c * CF::XT + 4 * q);
      }
      const float bias = bias_it[it][cc];
      const float2 b2 = make_float2(bias, bias);
      float2 x01 = __fadd2_rn(make_float2(dl.x, dl.y), b2);
      float2 x23 = __fadd2_rn(make_float2(dl.z, dl.w), b2);
      if (a.softplus) {
        x01 = softplus_fast2(x01);
        x23 = softplus_fast2(x23);
      }
      delt[cc][0] = x01.x;
      delt[cc][1] = x01.y;
      delt[cc][2] = x23.x;
      delt[cc][3] = x23.y;
      if constexpr (!kFull) {
        // padding steps and channels: A_bar = 1, B_bar u = 0 (state unchanged)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (d0 + c >= a.dim || t0 + 4 * q + k >= a.seqlen) delt[cc][k] = 0.f;
      }
      if (seg) dsum[it][cc] += (double)((delt[cc][0] + delt[cc][1]) + (delt[cc][2] + delt[cc][3]));
      const float2 w01 = __fmul2_rn(make_float2(delt[cc][0], delt[cc][1]), make_float2(uu.x, uu.y));
      const float2 w23 = __fmul2_rn(make_float2(delt[cc][2], delt[cc][3]), make_float2(uu.z, uu.w));
      w[cc][0] = w01.x;
      w[cc][1] = w01.y;
      w[cc][2] = w23.x;
      w[cc][3] = w23.y;
    }
    const int row = q * CF::DW_STRIDE + lg * CF::CPL;
    if constexpr (CF::CPL == 1) {
      dwD[row] = make_float4(delt[0][0], delt[0][1], delt[0][2], delt[0][3]);
      dwW[row] = make_float4(w[0][0], w[0][1], w[0][2], w[0][3]);
      if constexpr (CF::ZOH)  // 1/0 = inf on padding steps: the series branch of phi takes them
        dwI[row] = make_float4(rcp_approx(delt[0][0]), rcp_approx(delt[0][1]),
                               rcp_approx(delt[0][2]), rcp_approx(delt[0][3]));
    } else {  // the channel pair interleaved by step
      dwD[row] = make_float4(delt[0][0], delt[1][0], delt[0][1], delt[1][1]);
      dwD[row + 1] = make_float4(delt[0][2], delt[1][2], delt[0][3], delt[1][3]);
      dwW[row] = make_float4(w[0][0], w[1][0], w[0][1], w[1][1]);
      dwW[row + 1] = make_float4(w[0][2], w[1][2], w[0][3], w[1][3]);
    }
  }
  // B and C rows [n][t] -> [t][n/2 pairs][B_2p, B_2p+1, C_2p, C_2p+1]
  const E* rawB = raw + CF::OFF_B_T / CF::ES;
  const E* rawC = raw + CF::OFF_C_T / CF::ES;
  if constexpr (CF::ES == 2) {
    constexpr int TP = CF::T / 2;  // timestep pairs (one 32-bit word per row)
    const uint32_t* B32 = reinterpret_cast<const uint32_t*>(rawB);
    const uint32_t* C32 = reinterpret_cast<const uint32_t*>(rawC);
    constexpr int NB4 = CF::N / 4;
    // Item (tp, nb) reads rows 4 nb .. 4 nb + 3 at word tp.  The steps vary
    // fastest over the lanes, so a half-warp reads 16 consecutive words of a
    // row (with blocks fastest, every lane of a warp would read the same bank),
    // and the odd blocks take their rows in rotated order so that the two
    // half-warps read rows of opposite parity, i.e. opposite halves of the
    // banks.
    constexpr bool TP_FAST = CF::TP_FAST && TP == 16;
    for (int i = tid; i < NB4 * TP; i += CF::NT) {
      const int tp = TP_FAST ? i % TP : i / NB4;
      const int nb = TP_FAST ? i / TP : i - tp * NB4;
      const int rot = TP_FAST ? (nb & 1) : 0;
      uint32_t bv[4], cv4[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = 4 * nb + ((r + rot) & 3);
        bv[r] = B32[row * TP + tp];
        cv4[r] = C32[row * TP + tp];
      }
      uint32_t bw[4], cw[4];  // bw[k]: row 4 nb + k
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        bw[k] = rot ? bv[(k + 3) & 3] : bv[k];
        cw[k] = rot ? cv4[(k + 3) & 3] : cv4[k];
      }
      uint4* dst0 = reinterpret_cast<uint4*>(bc + (2 * tp) * CF::BC_ROW + CF::bc_pos(nb));
      uint4* dst1 = reinterpret_cast<uint4*>(bc + (2 * tp + 1) * CF::BC_ROW + CF::bc_pos(nb));
      *dst0 = make_uint4(__byte_perm(bw[0], bw[1], 0x5410), __byte_perm(cw[0], cw[1], 0x5410),
                         __byte_perm(bw[2], bw[3], 0x5410), __byte_perm(cw[2], cw[3], 0x5410));
      *dst1 = make_uint4(__byte_perm(bw[0], bw[1], 0x7632), __byte_perm(cw[0], cw[1], 0x7632),
                         __byte_perm(bw[2], bw[3], 0x7632), __byte_perm(cw[2], cw[3], 0x7632));
    }
  } else {
    const float* fb = reinterpret_cast<const float*>(rawB);
    const float* fc = reinterpret_cast<const float*>(rawC);
    for (int i = tid; i < (CF::N / 4) * CF::T; i += CF::NT) {
      const int nb = i / CF::T, t = i - nb * CF::T;
      unsigned char* row = bc + t * CF::BC_ROW;  // fp32: units 2 nb and 2 nb + 1
      *reinterpret_cast<float4*>(row + CF::bc_pos(2 * nb)) =
          make_float4(fb[(4 * nb) * CF::T + t], fb[(4 * nb + 1) * CF::T + t],
                      fc[(4 * nb) * CF::T + t], fc[(4 * nb + 1) * CF::T + t]);
      *reinterpret_cast<float4*>(row + CF::bc_pos(2 * nb + 1)) =
          make_float4(fb[(4 * nb + 2) * CF::T + t], fb[(4 * nb + 3) * CF::T + t],
                      fc[(4 * nb + 2) * CF::T + t], fc[(4 * nb + 3) * CF::T + t]);
    }
  }
}

// ------------------------------------------------------------- phase 2 ---

// B and C of NP consecutive state pairs at one timestep, as fp32 pairs; p
// points at the lane's first unit (16-byte loads where the pairs allow; the
// lane's next unit is UNIT_STRIDE bytes on).
template <class CF, int NP>
__device__ __forceinline__ void bc_pairs(const unsigned char* p, float2 (&b)[NP],
                                         float2 (&c)[NP]) {
  if constexpr (CF::BCES == 2) {
    if constexpr (NP % 2 == 0) {
#pragma unroll
      for (int i = 0; i < NP / 2; ++i) {
        const uint4 v = *reinterpret_cast<const uint4*>(p + i * CF::UNIT_STRIDE);
        b[2 * i] = bf16x2_to_float2(v.x);
        c[2 * i] = bf16x2_to_float2(v.y);
        b[2 * i + 1] = bf16x2_to_float2(v.z);
        c[2 * i + 1] = bf16x2_to_float2(v.w);
      }
    } else {
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const uint2 v = reinterpret_cast<const uint2*>(p)[i];
        b[i] = bf16x2_to_float2(v.x);
        c[i] = bf16x2_to_float2(v.y);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const float4 v = *reinterpret_cast<const float4*>(p + i * CF::UNIT_STRIDE);
      b[i] = make_float2(v.x, v.y);
      c[i] = make_float2(v.z, v.w);
    }
  }
}

// Exact zero-order hold: B_bar u = phi(x) Delta u B with x = Delta A (natural
// units) and phi(x) = (e^x - 1) / x = sum_k x^k / (k+1)!.  e = 2^(x log2 e) is
// the decay the recurrence already has.  Near x = 0, e - 1 cancels, so phi
// there comes from its Taylor series (in x2 = x log2 e, the argument of the
// ex2; the degree-5 truncation error is below 1e-8 for |x2| < kZohSeriesMax);
// elsewhere phi = (e - 1) (1/A) (1/Delta), whose rounding error is then below
// 2e-6 relative.  A select (not a blend) keeps A = 0 (1/A stored as 0) and
// padding steps (Delta = 0, 1/Delta = inf) on the series branch.
constexpr float kZohSeriesMax = 0.25f;
struct ZohSeries {  // phi(x2 ln 2) = sum_k c[k] x2^k, c[k] = ln2^k / (k+1)!
  static constexpr double ln2 = 0.69314718055994530942;
  __host__ __device__ static constexpr float c(int k) {
    double v = 1.0, f = 1.0;
    for (int i = 1; i <= k; ++i) {
      v *= ln2;
      f *= (double)(i + 1);
    }
    return (float)(v / f);
  }
};

__device__ __forceinline__ float zoh_phi(float x2, float e, float inv_a, float inv_dl) {
  constexpr float c0 = ZohSeries::c(0), c1 = ZohSeries::c(1), c2 = ZohSeries::c(2),
                  c3 = ZohSeries::c(3), c4 = ZohSeries::c(4), c5 = ZohSeries::c(5);
  float p = fmaf(c5, x2, c4);
  p = fmaf(p, x2, c3);
  p = fmaf(p, x2, c2);
  p = fmaf(p, x2, c1);
  p = fmaf(p, x2, c0);
  const float big = (e - 1.f) * inv_a * inv_dl;
  return fabsf(x2) < kZohSeriesMax ? p : big;
}

// The same on a pair of states (packed series and product, scalar selects).
__device__ __forceinline__ float2 zoh_phi2(float2 x2, float2 e, float2 inv_a, float2 inv_dl) {
  constexpr float c0 = ZohSeries::c(0), c1 = ZohSeries::c(1), c2 = ZohSeries::c(2),
                  c3 = ZohSeries::c(3), c4 = ZohSeries::c(4), c5 = ZohSeries::c(5);
  float2 p = __ffma2_rn(make_float2(c5, c5), x2, make_float2(c4, c4));
  p = __ffma2_rn(p, x2, make_float2(c3, c3));
  p = __ffma2_rn(p, x2, make_float2(c2, c2));
  p = __ffma2_rn(p, x2, make_float2(c1, c1));
  p = __ffma2_rn(p, x2, make_float2(c0, c0));
  const float2 big = __fmul2_rn(__fmul2_rn(__fadd2_rn(e, make_float2(-1.f, -1.f)), inv_a), inv_dl);
  return make_float2(fabsf(x2.x) < kZohSeriesMax ? p.x : big.x,
                     fabsf(x2.y) < kZohSeriesMax ? p.y : big.y);
}

// The recurrence for this lane's G states over the chunk, two states per
// packed fp32x2 operation.  Each lane writes its partial readout
// sum_{n in lane} C_t[n] h_t[n] for four timesteps at a time (one 16-byte
// store); phase 3 adds the K partials of a channel.  The time loop carries
// no cross-lane dependency, so the ex2 of later steps can issue while
// earlier steps' FMA chains drain.
template <class CF>
__device__ __forceinline__ void phase2(const float4* dwD, const float4* dwW, const float4* dwI,
                                       const unsigned char* bc, float* sy,
                                       float2 (&h)[CF::HP], const float2 (&a2)[CF::HP],
                                       const float2 (&ia)[CF::HP], int c, int j,
                                       const CkptCtx& ck) {
  constexpr int G2 = CF::G / 2;  // state pairs per lane
  // the lane's first unit (half units: G = 2 bf16 states, 8 bytes a lane)
  const unsigned char* bcj = bc + (CF::UPL >= 1 ? CF::bc_pos(j * CF::UPL) : j * G2 * CF::PAIR_BYTES);
  float* syr = sy + (c * CF::K + j) * CF::SY_STRIDE;
#pragma unroll kPhase2Unroll
  for (int q = 0; q < CF::QPR; ++q) {
    if (CF::TRAIN && ck.p && (q & 3) == 0 && 4 * q < ck.left) {  // the state before step 4q
      float2* dst = reinterpret_cast<float2*>(ck.p + (q >> 2) * ck.stride);
#pragma unroll
      for (int g = 0; g < CF::G / 2; ++g) dst[g] = h[g];
    }
    const float4 D4 = dwD[q * CF::DW_STRIDE + c];
    const float4 W4 = dwW[q * CF::DW_STRIDE + c];
    const float dls[4] = {D4.x, D4.y, D4.z, D4.w};
    const float ws[4] = {W4.x, W4.y, W4.z, W4.w};
    float idl[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (CF::ZOH) {
      const float4 I4 = dwI[q * CF::DW_STRIDE + c];
      idl[0] = I4.x; idl[1] = I4.y; idl[2] = I4.z; idl[3] = I4.w;
    }
    float s[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 dl2 = make_float2(dls[k], dls[k]);
      const float2 w2 = make_float2(ws[k], ws[k]);
      float2 bb[G2], cc[G2];
      bc_pairs<CF, G2>(bcj + (4 * q + k) * CF::BC_ROW, bb, cc);
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int g = 0; g < G2; ++g) {
        const float2 x = __fmul2_rn(dl2, a2[g]);
        const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        float2 wb;
        if constexpr (CF::ZOH)
          wb = __fmul2_rn(__fmul2_rn(zoh_phi2(x, e, ia[g], make_float2(idl[k], idl[k])), w2), bb[g]);
        else
          wb = __fmul2_rn(w2, bb[g]);
        h[g] = __ffma2_rn(e, h[g], wb);
        acc = __ffma2_rn(cc[g], h[g], acc);
      }
      s[k] = acc.x + acc.y;
    }
    *reinterpret_cast<float4*>(syr + 4 * q) = make_float4(s[0], s[1], s[2], s[3]);
  }
}

// The recurrence with two channels per lane (CPL = 2): the lane's G states n
// of channels c0 = 2 lg and c1 = 2 lg + 1 sit in G float2 registers
// {h_c0[n], h_c1[n]}, and each fp32x2 operation advances one state of both
// channels: A_bar = 2^({Delta_c0, Delta_c1} A log2 e), h = A_bar h + {w_c0, w_c1}
// B_t[n].  B_t[n] and C_t[n] are widened once and used for both channels; the
// partial readouts of the two channels go to their own rows of sy.
template <class CF>
__device__ __forceinline__ void phase2_cpl2(const float4* dwD, const float4* dwW,
                                            const unsigned char* bc, float* sy,
                                            float2 (&h)[CF::HP], const float2 (&a2)[CF::HP],
                                            int lg, int j) {
  constexpr int G = CF::G;
  const unsigned char* bcj = bc + CF::bc_pos(j * CF::UPL);
  float* sy0 = sy + (2 * lg * CF::K + j) * CF::SY_STRIDE;
  float* sy1 = sy0 + CF::K * CF::SY_STRIDE;
#pragma unroll kPhase2Unroll
  for (int q = 0; q < CF::QPR; ++q) {
    const int row = q * CF::DW_STRIDE + 2 * lg;
    const float4 D01 = dwD[row], D23 = dwD[row + 1];
    const float4 W01 = dwW[row], W23 = dwW[row + 1];
    const float2 dls[4] = {make_float2(D01.x, D01.y), make_float2(D01.z, D01.w),
                           make_float2(D23.x, D23.y), make_float2(D23.z, D23.w)};
    const float2 ws[4] = {make_float2(W01.x, W01.y), make_float2(W01.z, W01.w),
                          make_float2(W23.x, W23.y), make_float2(W23.z, W23.w)};
    float s0[4], s1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float2 bb[G / 2], cc[G / 2];
      bc_pairs<CF, G / 2>(bcj + (4 * q + k) * CF::BC_ROW, bb, cc);
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int n = 0; n < G; ++n) {
        const float bn = (n & 1) ? bb[n >> 1].y : bb[n >> 1].x;
        const float cn = (n & 1) ? cc[n >> 1].y : cc[n >> 1].x;
        const float2 x = __fmul2_rn(dls[k], a2[n]);
        const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        const float2 wb = make_float2(ws[k].x * bn, ws[k].y * bn);
        h[n] = __ffma2_rn(e, h[n], wb);
        acc0 = fmaf(cn, h[n].x, acc0);
        acc1 = fmaf(cn, h[n].y, acc1);
      }
      s0[k] = acc0;
      s1[k] = acc1;
    }
    *reinterpret_cast<float4*>(sy0 + 4 * q) = make_float4(s0[0], s0[1], s0[2], s0[3]);
    *reinterpret_cast<float4*>(sy1 + 4 * q) = make_float4(s1[0], s1[1], s1[2], s1[3]);
  }
}

// The time-split recurrence (WT > 1).  Warp wt scans steps
// [wt TW, (wt+1) TW) of the chunk from h = 0 while tracking the product of
// its decays P_t = prod A_bar and the fix-up coefficients Q_t = C_t P_t; the
// WT warps then swap their aggregates (P_end, h_end) through shared memory and
// each folds the chunk's carry-in through the aggregates before it with the
// operator (a1,b1) then (a2,b2) = (a2 a1, a2 b1 + b2) ("Mamba 选择性机制",
// sec. 3.1), which gives its own carry-in h_in exactly: h_t = local h_t +
// P_t h_in, so the readout is corrected by sum_n Q_t[n] h_in[n].  Every warp
// folds all WT aggregates, so all of them leave with the chunk's carry-out in
// h.  No ex2 is evaluated twice.
template <class CF>
__device__ __forceinline__ void phase2_split(const float4* dwD, const float4* dwW,
                                             const float4* dwI, const unsigned char* bc,
                                             float* sy, float* aggP, float* aggH,
                                             float2 (&h)[CF::HP], const float2 (&a2)[CF::HP],
                                             const float2 (&ia)[CF::HP], int c, int j, int wt,
                                             int lane_g, const CkptCtx& ck) {
  constexpr int G2 = CF::G / 2;
  const unsigned char* bcj = bc + (CF::UPL >= 1 ? CF::bc_pos(j * CF::UPL) : j * G2 * CF::PAIR_BYTES);
  float2 hl[G2], P[G2];
#pragma unroll
  for (int g = 0; g < G2; ++g) {
    hl[g] = make_float2(0.f, 0.f);
    P[g] = make_float2(1.f, 1.f);
  }
  float2 Q[CF::TW][G2];
  float s[CF::TW];
#pragma unroll
  for (int q = 0; q < CF::TW / 4; ++q) {
    const int qq = wt * (CF::TW / 4) + q;
    const float4 D4 = dwD[qq * CF::DW_STRIDE + c];
    const float4 W4 = dwW[qq * CF::DW_STRIDE + c];
    const float dls[4] = {D4.x, D4.y, D4.z, D4.w};
    const float ws[4] = {W4.x, W4.y, W4.z, W4.w};
    float idl[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (CF::ZOH) {
      const float4 I4 = dwI[qq * CF::DW_STRIDE + c];
      idl[0] = I4.x; idl[1] = I4.y; idl[2] = I4.z; idl[3] = I4.w;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = 4 * q + k;
      const unsigned char* row = bcj + (4 * qq + k) * CF::BC_ROW;
      const float2 dl2 = make_float2(dls[k], dls[k]);
      const float2 w2 = make_float2(ws[k], ws[k]);
      float2 acc = make_float2(0.f, 0.f);
      float2 bb[G2], cc[G2];
      bc_pairs<CF, G2>(row, bb, cc);
#pragma unroll
      for (int g = 0; g < G2; ++g) {
        const float2 x = __fmul2_rn(dl2, a2[g]);
        const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        float2 wb;
        if constexpr (CF::ZOH)
          wb = __fmul2_rn(__fmul2_rn(zoh_phi2(x, e, ia[g], make_float2(idl[k], idl[k])), w2), bb[g]);
        else
          wb = __fmul2_rn(w2, bb[g]);
        hl[g] = __ffma2_rn(e, hl[g], wb);
        P[g] = __fmul2_rn(e, P[g]);
        acc = __ffma2_rn(cc[g], hl[g], acc);
        Q[t][g] = __fmul2_rn(cc[g], P[g]);
      }
      s[t] = acc.x + acc.y;
    }
  }
  // publish this warp's aggregate: [wt][lane in channel set][state]
  float2* myP = reinterpret_cast<float2*>(aggP + (wt * CF::WC * 32 + lane_g) * CF::G);
  float2* myH = reinterpret_cast<float2*>(aggH + (wt * CF::WC * 32 + lane_g) * CF::G);
#pragma unroll
  for (int g = 0; g < G2; ++g) {
    myP[g] = P[g];
    myH[g] = hl[g];
  }
  __syncthreads();
  float2 hin[G2];
#pragma unroll
  for (int v = 0; v < CF::WT; ++v) {
    if (v == wt) {
#pragma unroll
      for (int g = 0; g < G2; ++g) hin[g] = h[g];
    }
    const float2* vP = reinterpret_cast<const float2*>(aggP + (v * CF::WC * 32 + lane_g) * CF::G);
    const float2* vH = reinterpret_cast<const float2*>(aggH + (v * CF::WC * 32 + lane_g) * CF::G);
#pragma unroll
    for (int g = 0; g < G2; ++g) h[g] = __ffma2_rn(vP[g], h[g], vH[g]);
  }
  // hin is the state before this warp's first step: a 16-step checkpoint when
  // the segment starts on one
  if (CF::TRAIN && ck.p && (wt * CF::TW) % 16 == 0 && wt * CF::TW < ck.left) {
    float2* dst = reinterpret_cast<float2*>(ck.p + (wt * CF::TW / 16) * ck.stride);
#pragma unroll
    for (int g = 0; g < G2; ++g) dst[g] = hin[g];
  }
  float* syr = sy + (c * CF::K + j) * CF::SY_STRIDE + wt * CF::TW;
#pragma unroll
  for (int q = 0; q < CF::TW / 4; ++q) {
    float out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = 4 * q + k;
      float2 fix = make_float2(0.f, 0.f);
#pragma unroll
      for (int g = 0; g < G2; ++g) fix = __ffma2_rn(Q[t][g], hin[g], fix);
      out[k] = s[t] + (fix.x + fix.y);
    }
    *reinterpret_cast<float4*>(syr + 4 * q) = make_float4(out[0], out[1], out[2], out[3]);
  }
}

// ------------------------------------------------------------- phase 3 ---

template <class CF, bool kFull>
__device__ __forceinline__ void phase3(const FwdArgs& a, const typename CF::Elem* raw,
                                       const float* sy, const float4* su,
                                       const float (&D_it)[CF::ITEMS_PER_THREAD], int64_t b,
                                       int64_t d0, int64_t t0, bool has_z) {
  const int64_t L = a.seqlen, D = a.dim;
  const int tid = threadIdx.x;
  const typename CF::Elem* rawZ = raw + CF::OFF_Z_T / CF::ES;
#pragma unroll
  for (int it = 0; it < CF::ITEMS_PER_THREAD; ++it) {
    const int i = tid + it * CF::NT;
    if (CF::ITEM_GUARD && i >= CF::ITEMS) break;
    const int c = i / CF::QPR, q = i - c * CF::QPR;
    const int64_t d = d0 + c, t = t0 + 4 * q;
    if constexpr (!kFull) {
      if (d >= D || t >= L) continue;
    }
    const float4 s0 = *reinterpret_cast<const float4*>(sy + (c * CF::K) * CF::SY_STRIDE + 4 * q);
    float2 s01 = make_float2(s0.x, s0.y), s23 = make_float2(s0.z, s0.w);
#pragma unroll
    for (int jj = 1; jj < CF::K; ++jj) {
      const float4 o = *reinterpret_cast<const float4*>(sy + (c * CF::K + jj) * CF::SY_STRIDE + 4 * q);
      s01 = __fadd2_rn(s01, make_float2(o.x, o.y));
      s23 = __fadd2_rn(s23, make_float2(o.z, o.w));
    }
    float4 uu;
    if constexpr (CF::CONV) uu = su[q * CF::DW_STRIDE + c];
    else uu = load4_f32(raw + c * CF::XT + 4 * q);
    const float Dd = D_it[it];
    const float2 D2 = make_float2(Dd, Dd);
    float2 y01 = __ffma2_rn(D2, make_float2(uu.x, uu.y), s01);
    float2 y23 = __ffma2_rn(D2, make_float2(uu.z, uu.w), s23);
    if (has_z) {
      const float4 zz = load4_f32(rawZ + c * CF::T + 4 * q);
      y01 = __fmul2_rn(y01, silu_fast2(make_float2(zz.x, zz.y)));
      y23 = __fmul2_rn(y23, silu_fast2(make_float2(zz.z, zz.w)));
    }
    const float y[4] = {y01.x, y01.y, y23.x, y23.y};
    const int64_t iy = (b * D + d) * L + t;
    float* dst = a.y + iy;
    if (a.vec && (kFull || t + 3 < L)) {  // 16-byte stores only on aligned rows
      if (in_range(iy, 4, a.batch * D * L))
        *reinterpret_cast<float4*>(dst) = make_float4(y[0], y[1], y[2], y[3]);
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (t + k < L && in_range(iy + k, a.batch * D * L)) dst[k] = y[k];
    }
  }
}

// ------------------------------------------------------------ schedule ---

// Work is the sequence of (channel group, chunk) units, group-major; worker w
// (one CTA) owns units [w U / W, (w+1) U / W).  A range can start inside a
// group (its "suffix" piece needs the state at that chunk from worker w-1)
// and end inside a group (its "prefix" piece hands its final state to worker
// w+1).  Each worker runs its prefix piece first (it starts from h = 0 and
// publishes as early as possible), then its whole groups, then its suffix
// piece, so the carry it waits for was produced at the very start of its
// predecessor's run.  The host keeps every range at least one group long, so
// no piece needs a carry in and hands one out at once.
struct Sched {
  int64_t units;        // groups x chunks per group
  int64_t nk;           // chunks per group
  int64_t tiles_per_b;  // channel tiles per batch row
  float* carries;       // [workers][CH * N] published prefix states (nullable)
  unsigned long long* flags;  // [workers] epoch of the published carry
  unsigned long long epoch;   // unique per launch, so stale flags never match
  unsigned int* ticket;       // balanced schedule: worker-id counter, 0 at launch
  uint32_t spin_limit;        // polls before a carry wait gives up
  int skip_publish;           // test hook: this worker never publishes (-1: none)
  // plain schedule only: each channel group's chunks are cut into nseg
  // segments of seg_chunks chunks (the last may be shorter), one CTA each
  int32_t nseg;
  int64_t seg_chunks;
};

// Walks one worker's chunk sequence without divisions: the three pieces
// (prefix, whole groups, suffix) are set up once per CTA; advancing is a few
// compares.  All fields are uniform across the CTA.
struct Cursor {
  int32_t g, c;        // channel group, chunk index within the group
  int32_t b, tile;     // batch row, channel tile of group g
  int32_t piece;       // 0 prefix, 1 whole groups, 2 suffix, 3 done
  int64_t left;        // chunks left in the current piece
  int64_t len;         // length of the current piece
  // piece descriptors (same for every cursor of the CTA); scalars, so that
  // nothing here is indexed at run time
  int32_t g0, g1, g2, c2;
  int64_t n0, n1, n2;
  int32_t nk, tiles;

  __device__ __forceinline__ void seat(int32_t gg, int32_t cc) {
    g = gg;
    c = cc;
    b = gg / tiles;  // only when a piece starts
    tile = gg - b * tiles;
  }
  __device__ __forceinline__ void enter(int32_t p) {
    if (p == 0 && n0 == 0) p = 1;
    if (p == 1 && n1 == 0) p = 2;
    if (p == 2 && n2 == 0) p = 3;
    piece = p;
    if (p == 0) { len = n0; seat(g0, 0); }
    else if (p == 1) { len = n1; seat(g1, 0); }
    else if (p == 2) { len = n2; seat(g2, c2); }
    left = len;
  }
  __device__ __forceinline__ void init(const Sched& s, int64_t u0, int64_t u1) {
    nk = (int32_t)s.nk;
    tiles = (int32_t)s.tiles_per_b;
    const int64_t gfull0 = (u0 + s.nk - 1) / s.nk;
    g0 = (int32_t)(u1 / s.nk);  n0 = u1 % s.nk;
    g1 = (int32_t)gfull0;       n1 = (u1 / s.nk - gfull0) * s.nk;
    g2 = (int32_t)(u0 / s.nk);  c2 = (int32_t)(u0 % s.nk);
    n2 = c2 ? s.nk - c2 : 0;
    enter(0);
  }
  __device__ __forceinline__ void advance() {
    if (--left == 0) {
      enter(piece + 1);
      return;
    }
    if (++c == nk) {
      c = 0;
      ++g;
      if (++tile == tiles) {
        tile = 0;
        ++b;
      }
    }
  }
  __device__ __forceinline__ bool first() const { return c == 0 || left == len; }
  __device__ __forceinline__ bool carry_in() const { return piece == 2 && left == len; }
  __device__ __forceinline__ bool carry_out() const { return piece == 0 && left == 1; }
  __device__ __forceinline__ bool last() const { return c == nk - 1; }
};

// Bounded wait for worker `src`'s carry of this launch (one thread).  The
// consumer clears the flag it took: each flag has one consumer, so a replay of
// the same launch (a captured CUDA graph keeps its epoch) never mistakes the
// previous replay's flag for a fresh carry.
__device__ __forceinline__ bool wait_carry(const Sched& s, int src) {
  if (!in_range(src, gridDim.x)) return false;
  unsigned long long* f = s.flags + src;
  for (uint32_t i = 0; i < s.spin_limit; ++i) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];\n" : "=l"(v) : "l"(f) : "memory");
    if (v == s.epoch) {
      asm volatile("st.relaxed.gpu.global.u64 [%0], %1;\n" ::"l"(f), "l"(0ull) : "memory");
      return true;
    }
    __nanosleep(i < 64 ? 32 : 256);
  }
  atomicOr(&g_error_word, kErrLookback);
  return false;
}

__device__ __forceinline__ void publish_carry(const Sched& s, int w) {
  if (!in_range(w, gridDim.x)) return;
  unsigned long long* f = s.flags + w;
  asm volatile("st.release.gpu.global.u64 [%0], %1;\n" ::"l"(f), "l"(s.epoch) : "memory");
}

// A lane's decay constants for states n, n+1 of channel d: A log2 e (the ex2
// argument per unit Delta) and, for the exact zero-order hold, 1/A (0 where
// A = 0, which the series branch covers).
template <class CF>
__device__ __forceinline__ void load_decay(const FwdArgs& a, int64_t d, int n, bool chan_ok,
                                           float2& a2, float2& ia) {
  const bool in = chan_ok && in_range(d * CF::N + n, 2, a.dim * CF::N);
  const float A0 = in ? __ldg(a.A + d * CF::N + n) : 0.f;
  const float A1 = in ? __ldg(a.A + d * CF::N + n + 1) : 0.f;
  a2 = make_float2(A0 * 1.4426950408889634f, A1 * 1.4426950408889634f);
  ia = CF::ZOH ? make_float2(A0 != 0.f ? 1.f / A0 : 0.f, A1 != 0.f ? 1.f / A1 : 0.f)
               : make_float2(0.f, 0.f);
}

// This thread's convolution taps for its items of channel tile d0, placed
// right-aligned in kConvTaps slots (zeros before a shorter filter).
template <class CF>
__device__ __forceinline__ void load_conv_regs(const FwdArgs& a, int64_t d0, ConvRegs<CF>& cv) {
  if constexpr (CF::CONV) {
    const int W = a.conv_width;
#pragma unroll
    for (int it = 0; it < CF::ITEMS1_PER_THREAD; ++it) {
      const int64_t d = d0 + (threadIdx.x + it * CF::NT) / CF::QPR;
      const bool ok = d < a.dim;
#pragma unroll
      for (int k = 0; k < kConvTaps; ++k) {
        const int src = k - (kConvTaps - W);
        cv.w[it][k] = (ok && src >= 0 && in_range(d * W + src, a.dim * W)) ? __ldg(a.conv_w + d * W + src) : 0.f;
      }
      cv.b[it] = (ok && a.conv_b) ? __ldg(a.conv_b + d) : 0.f;
    }
  }
}

// A lane's states of its CPL channels as HP float2 registers (see phase2 and
// phase2_cpl2 for the packing), read from or written to [channel][N] fp32
// rows; row(cc) gives the row of the lane's channel cc, or null (zeros; not
// written).
template <class CF, class RowFn>
__device__ __forceinline__ void lane_load_state(float2 (&h)[CF::HP], RowFn row, int j) {
  if constexpr (CF::CPL == 1) {
    const float* r = row(0);
#pragma unroll
    for (int g = 0; g < CF::HP; ++g) {
      const int n = j * CF::G + 2 * g;
      h[g] = r ? make_float2(r[n], r[n + 1]) : make_float2(0.f, 0.f);
    }
  } else {
    const float* r0 = row(0);
    const float* r1 = row(1);
#pragma unroll
    for (int g = 0; g < CF::HP; ++g) {
      const int n = j * CF::G + g;
      h[g] = make_float2(r0 ? r0[n] : 0.f, r1 ? r1[n] : 0.f);
    }
  }
}

template <class CF, class RowFn>
__device__ __forceinline__ void lane_store_state(const float2 (&h)[CF::HP], RowFn row, int j) {
  if constexpr (CF::CPL == 1) {
    float* r = row(0);
    if (r)
#pragma unroll
      for (int g = 0; g < CF::HP; ++g) {
        const int n = j * CF::G + 2 * g;
        r[n] = h[g].x;
        r[n + 1] = h[g].y;
      }
  } else {
    float* r0 = row(0);
    float* r1 = row(1);
#pragma unroll
    for (int g = 0; g < CF::HP; ++g) {
      const int n = j * CF::G + g;
      if (r0) r0[n] = h[g].x;
      if (r1) r1[n] = h[g].y;
    }
  }
}

// The lane's decay constants A log2 e (and 1/A for the exact zero-order hold)
// for channels d0 + lg CPL + cc, packed like its states (zeros past dim).
template <class CF>
__device__ __forceinline__ void lane_load_decay(const FwdArgs& a, int64_t d0, int lg, int j,
                                                float2 (&a2)[CF::HP], float2 (&ia)[CF::HP]) {
  if constexpr (CF::CPL == 1) {
    const int64_t d = d0 + lg;
#pragma unroll
    for (int g = 0; g < CF::HP; ++g) load_decay<CF>(a, d, j * CF::G + 2 * g, d < a.dim, a2[g], ia[g]);
  } else {
    const int64_t e0 = d0 + 2 * lg, e1 = e0 + 1;
#pragma unroll
    for (int g = 0; g < CF::HP; ++g) {
      const int n = j * CF::G + g;
      const float A0 = (e0 < a.dim && in_range(e0 * CF::N + n, a.dim * CF::N)) ? __ldg(a.A + e0 * CF::N + n) : 0.f;
      const float A1 = (e1 < a.dim && in_range(e1 * CF::N + n, a.dim * CF::N)) ? __ldg(a.A + e1 * CF::N + n) : 0.f;
      a2[g] = make_float2(A0 * 1.4426950408889634f, A1 * 1.4426950408889634f);
      ia[g] = make_float2(0.f, 0.f);
    }
  }
}

// -------------------------------------------------------------- kernel ---

// kMulti = false: one channel group (or one segment of its sequence) per CTA,
// a plain loop over its chunks.  kMulti = true: balanced ranges with carry
// handoff.
template <class CF, bool kMulti>
__global__ void __launch_bounds__(CF::NT, CF::MIN_CTAS)
    scan_fwd_chunked_kernel(const FwdArgs a, const __grid_constant__ FwdMaps maps,
                            const Sched sched) {
  using E = typename CF::Elem;
  constexpr int HP = CF::HP, CPL = CF::CPL;
  extern __shared__ __align__(128) unsigned char smem_dyn[];
  // TMA destinations want 128-byte alignment; the dynamic window follows the
  // static arrays, so align its base explicitly (SMEM_BYTES has the slack).
  unsigned char* smem = smem_dyn + ((128u - (smem_u32(smem_dyn) & 127u)) & 127u);
  // stage j & 1 of the raw tiles (pointer arithmetic: no indexed local array)
  auto raw = [&](int64_t j) { return smem + (j & 1) * CF::OFF_RAW1; };
  float4* dwD = reinterpret_cast<float4*>(smem + CF::OFF_DWD);
  float4* dwW = reinterpret_cast<float4*>(smem + CF::OFF_DWW);
  unsigned char* bc = smem + CF::OFF_BC;
  float* sy = reinterpret_cast<float*>(smem + CF::OFF_SY);
  float4* su = reinterpret_cast<float4*>(smem + CF::OFF_SU);    // CONV only
  float4* dwI = reinterpret_cast<float4*>(smem + CF::OFF_DWI);  // ZOH only
  float* aggP = reinterpret_cast<float*>(smem + CF::OFF_AGG);     // time split only
  float* aggH = aggP + CF::AGG_FLOATS;
  __shared__ __align__(8) uint64_t bars[2];

  // kMulti: the worker id is the CTA's place in the order in which CTAs
  // started (an atomic ticket), not blockIdx.x: worker w - 1, whose carry
  // worker w waits for, then always runs already, whatever else holds SM slots.
  int w = blockIdx.x;
  if constexpr (kMulti) {
    __shared__ int sh_ticket;
    if (threadIdx.x == 0) sh_ticket = (int)atomicAdd(sched.ticket, 1u);
    __syncthreads();
    w = sh_ticket;
    if (!in_range(w, gridDim.x)) return;
  }
  // kMulti: worker w's range of (group, chunk) units; plain: CTA w runs
  // segment `seg` (chunks c_begin .. c_begin + nseq - 1) of channel group `grp`
  int64_t u0 = 0, u1 = 0, nseq = 0, c_begin = 0, grp = w;
  int seg = 0;
  if constexpr (kMulti) {
    u0 = sched.units * w / gridDim.x;
    u1 = sched.units * (w + 1) / gridDim.x;
    nseq = u1 - u0;
  } else {
    grp = w / sched.nseg;
    seg = (int)(w - grp * sched.nseg);
    c_begin = (int64_t)seg * sched.seg_chunks;
    nseq = sched.nk - c_begin < sched.seg_chunks ? sched.nk - c_begin : sched.seg_chunks;
  }
  const int64_t L = a.seqlen;
  const bool has_z = a.z != nullptr;
  const bool tma = a.vec != 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wc = warp % CF::WC, wt = warp / CF::WC;  // channel warp, time-split slot
  const int lg = wc * CF::LGW + lane / CF::K;  // this lane's group: channels lg CPL + cc
  const int j = lane % CF::K;                  // this lane's state group
  const int lane_g = wc * 32 + lane;           // lane within its channel set (time split)
  const bool writer = wt == 0;  // time-split warps hold the same carry: one writes it
  const int64_t ck_nk = (a.seqlen + 15) / 16;
  // this lane's checkpoint slot for the chunk of batch row bb starting at t0
  // (training variant, one channel per lane)
  auto ckpt_at = [&](int64_t bb, int64_t dd, bool ok, int64_t t0) {
    CkptCtx ck;
    ck.stride = a.dim * CF::N;
    ck.left = a.seqlen - t0;
    // this chunk's checkpoints: every 16th step while steps remain
    const int64_t i0 = ((bb * ck_nk + t0 / 16) * a.dim + dd) * CF::N + j * CF::G;
    const int64_t nck = (ck.left + 15) / 16 < CF::T / 16 ? (ck.left + 15) / 16 : CF::T / 16;
    ck.p = (CF::TRAIN && a.ckpt && ok &&
            in_range(i0 + (nck - 1) * ck.stride, CF::G, a.batch * ck_nk * a.dim * CF::N))
               ? a.ckpt + i0
               : nullptr;
    return ck;
  };
  auto run_phase2 = [&](float2 (&hh)[HP], const float2 (&aa)[HP], const float2 (&ii)[HP],
                        const CkptCtx& ck) {
    if constexpr (CF::WT > 1)
      phase2_split<CF>(dwD, dwW, dwI, bc, sy, aggP, aggH, hh, aa, ii, lg, j, wt, lane_g, ck);
    else if constexpr (CPL == 1)
      phase2<CF>(dwD, dwW, dwI, bc, sy, hh, aa, ii, lg, j, ck);
    else
      phase2_cpl2<CF>(dwD, dwW, bc, sy, hh, aa, lg, j);
  };
  // [channel][N] rows of this lane's channels in a per-(b, d) array, for batch
  // row bb of channel tile d0 (null past dim)
  auto rows_in = [&](float* base, int64_t bb, int64_t d0) {
    return [=](int cc) -> float* {
      const int64_t d = d0 + lg * CPL + cc;
      return (base && d < a.dim && in_range((bb * a.dim + d) * CF::N, CF::N, a.batch * a.dim * CF::N))
                 ? base + (bb * a.dim + d) * CF::N
                 : nullptr;
    };
  };
  // per-item constants: bias per (phase-1 item, channel), D per phase-3 item
  auto load_bias = [&](int64_t d0, float (&dst)[CF::ITEMS1_PER_THREAD][CPL]) {
#pragma unroll
    for (int it = 0; it < CF::ITEMS1_PER_THREAD; ++it)
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) {
        const int64_t d = d0 + ((tid + it * CF::NT) / CF::QPR) * CPL + cc;
        dst[it][cc] = (a.delta_bias && d < a.dim) ? __ldg(a.delta_bias + d) : 0.f;
      }
  };
  auto load_D = [&](int64_t d0, float (&dst)[CF::ITEMS_PER_THREAD]) {
#pragma unroll
    for (int it = 0; it < CF::ITEMS_PER_THREAD; ++it) {
      const int64_t d = d0 + (tid + it * CF::NT) / CF::QPR;
      dst[it] = (a.D && d < a.dim) ? __ldg(a.D + d) : 0.f;
    }
  };

  if (tma && tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (nseq <= 0) return;

  if constexpr (!kMulti) {
    // ---- one channel group (or one segment of it) per CTA: local chunk k is
    // chunk c_begin + k of the group ----
    const int64_t b = grp / sched.tiles_per_b;
    const int64_t d0 = (grp - b * sched.tiles_per_b) * CF::CH;
    const bool full_tile = d0 + CF::CH <= a.dim;
    const bool segmented = sched.nseg > 1;
    float bias_it[CF::ITEMS1_PER_THREAD][CPL], D_it[CF::ITEMS_PER_THREAD];
    double dsum[CF::ITEMS1_PER_THREAD][CPL];
    ConvRegs<CF> cv;
    load_bias(d0, bias_it);
    load_D(d0, D_it);
#pragma unroll
    for (int it = 0; it < CF::ITEMS1_PER_THREAD; ++it)
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) dsum[it][cc] = 0.0;
    load_conv_regs<CF>(a, d0, cv);
    float2 h[HP], a2[HP], ia[HP];
    // plain loads: h0 may be the last_state buffer this kernel writes; only
    // the first segment starts from it (later ones start from zero)
    lane_load_state<CF>(h, rows_in(seg == 0 ? const_cast<float*>(a.h0) : nullptr, b, d0), j);
    lane_load_decay<CF>(a, d0, lg, j, a2, ia);
    const int64_t d_ck = d0 + lg;  // training variant: the lane's channel
    bool ok = true;
    auto t_of = [&](int64_t k) { return (c_begin + k) * CF::T; };
    auto full_chunk = [&](int64_t k) { return full_tile && t_of(k) + CF::T <= L; };
    auto stage_in = [&](int64_t k) {
      if (tma) ok = ok && mbar_wait_bounded(&bars[k & 1], (uint32_t)((k >> 1) & 1), kTmaSpinLimit);
      else load_chunk_scalar<CF>(a, reinterpret_cast<E*>(raw(k)), b, d0, t_of(k));
    };
    auto run_phase1 = [&](int64_t k) {
      const E* rp = reinterpret_cast<const E*>(raw(k));
      if (full_chunk(k))
        phase1<CF, true>(a, rp, dwD, dwW, dwI, su, bc, bias_it, cv, d0, t_of(k), dsum, segmented);
      else
        phase1<CF, false>(a, rp, dwD, dwW, dwI, su, bc, bias_it, cv, d0, t_of(k), dsum, segmented);
    };
    auto drain = [&](int64_t first, int64_t last) {
      if (tma)
        for (int64_t kk = first; kk <= last && kk < nseq; ++kk)
          mbar_wait_bounded(&bars[kk & 1], (uint32_t)((kk >> 1) & 1), kTmaSpinLimit);
    };
    if (tma && tid == 0) {
      tma_chunk<CF>(maps, raw(0), &bars[0], (int32_t)b, (int32_t)d0, (int32_t)t_of(0), has_z);
      if (nseq > 1) tma_chunk<CF>(maps, raw(1), &bars[1], (int32_t)b, (int32_t)d0, (int32_t)t_of(1), has_z);
    }
    stage_in(0);
    if (!__syncthreads_and(ok)) {
      drain(0, 1);
      return;
    }
    run_phase1(0);
    __syncthreads();
    for (int64_t k = 0; k < nseq; ++k) {
      run_phase2(h, a2, ia, ckpt_at(b, d_ck, d_ck < a.dim, t_of(k)));
      if (k + 1 < nseq) stage_in(k + 1);
      if (!__syncthreads_and(ok)) {
        drain(k + 1, k + 1);
        return;
      }
      const E* rc = reinterpret_cast<const E*>(raw(k));
      if (full_chunk(k)) phase3<CF, true>(a, rc, sy, su, D_it, b, d0, t_of(k), has_z);
      else phase3<CF, false>(a, rc, sy, su, D_it, b, d0, t_of(k), has_z);
      if (k + 1 < nseq) run_phase1(k + 1);
      __syncthreads();
      if (tma && tid == 0 && k + 2 < nseq)
        tma_chunk<CF>(maps, raw(k), &bars[k & 1], (int32_t)b, (int32_t)d0, (int32_t)t_of(k + 2), has_z);
    }
    if (segmented) {
      // this segment's end state (from h = 0 unless it is the first) and its
      // sum of Delta; the carry-in correction pass combines them
      if (writer) lane_store_state<CF>(h, [&](int cc) -> float* {
        const int64_t d = d0 + lg * CPL + cc;
        const int64_t i0 = ((b * a.dim + d) * sched.nseg + seg) * CF::N;
        return (d < a.dim && in_range(i0, CF::N, a.batch * a.dim * sched.nseg * CF::N))
                   ? a.seg_h + i0
                   : nullptr;
      }, j);
      // the QPR threads of a phase-1 item are consecutive lanes of one warp
#pragma unroll
      for (int it = 0; it < CF::ITEMS1_PER_THREAD; ++it)
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) {
          double v = dsum[it][cc];
#pragma unroll
          for (int o = 1; o < CF::QPR; o <<= 1) v += __shfl_xor_sync(kFullMask, v, o);
          const int i = tid + it * CF::NT;
          const int64_t di = d0 + (i / CF::QPR) * CPL + cc;
          const int64_t is = (b * a.dim + di) * sched.nseg + seg;
          if ((i % CF::QPR) == 0 && i < CF::ITEMS1 && di < a.dim &&
              in_range(is, a.batch * a.dim * sched.nseg))
            a.seg_dsum[is] = (float)v;
        }
    } else if (writer) {
      lane_store_state<CF>(h, rows_in(a.last_state, b, d0), j);
    }
    return;
  }

  // three cursors over the same sequence: the chunk in the recurrence (cur),
  // the one being prepared (prep, one ahead) and the one being fetched (fetch)
  Cursor cur, prep, fetch;
  cur.init(sched, u0, u1);
  prep = cur;
  fetch = cur;

  float2 h[HP], a2[HP], ia[HP];
  float bias_it[CF::ITEMS1_PER_THREAD][CPL], D_it[CF::ITEMS_PER_THREAD];
  double no_dsum[CF::ITEMS1_PER_THREAD][CPL];  // (unused: the balanced schedule has no segments)
  ConvRegs<CF> cv;
  int32_t bias_g = -1, D_g = -1;  // group whose bias (and taps) / D are cached
  bool ok = true;  // false once a bounded wait has given up (error word set)

  auto d0_of = [&](const Cursor& r) { return (int64_t)r.tile * CF::CH; };
  auto full_chunk = [&](const Cursor& r) {
    return d0_of(r) + CF::CH <= a.dim && ((int64_t)r.c + 1) * CF::T <= L;
  };
  auto issue = [&](int64_t jj) {  // one thread: TMA loads of sequence chunk jj (= fetch)
    tma_chunk<CF>(maps, raw(jj), &bars[jj & 1], fetch.b, (int32_t)d0_of(fetch), fetch.c * CF::T,
                  has_z);
  };
  auto stage_in = [&](int64_t jj, const Cursor& r) {  // make chunk jj resident in raw(jj)
    if (tma) {
      ok = ok && mbar_wait_bounded(&bars[jj & 1], (uint32_t)((jj >> 1) & 1), kTmaSpinLimit);
    } else {
      load_chunk_scalar<CF>(a, reinterpret_cast<E*>(raw(jj)), r.b, d0_of(r), (int64_t)r.c * CF::T);
    }
  };
  auto run_phase1 = [&](int64_t jj) {  // jj = prep's chunk
    if (prep.g != bias_g) {
      load_bias(d0_of(prep), bias_it);
      load_conv_regs<CF>(a, d0_of(prep), cv);
      bias_g = prep.g;
    }
    const E* rp = reinterpret_cast<const E*>(raw(jj));
    const int64_t t0 = (int64_t)prep.c * CF::T;
    if (full_chunk(prep))
      phase1<CF, true>(a, rp, dwD, dwW, dwI, su, bc, bias_it, cv, d0_of(prep), t0, no_dsum, false);
    else
      phase1<CF, false>(a, rp, dwD, dwW, dwI, su, bc, bias_it, cv, d0_of(prep), t0, no_dsum, false);
  };
  // On a timed-out wait: wait (bounded) for every copy this CTA still has in
  // flight, so that none lands in shared memory after the CTA has left.
  auto drain = [&](int64_t first, int64_t last) {
    if (tma)
      for (int64_t kk = first; kk <= last && kk < nseq; ++kk)
        mbar_wait_bounded(&bars[kk & 1], (uint32_t)((kk >> 1) & 1), kTmaSpinLimit);
  };

  if (tma && tid == 0) {
    issue(0);
    fetch.advance();
    if (nseq > 1) {
      issue(1);
      fetch.advance();
    }
  }
  stage_in(0, prep);
  if (!__syncthreads_and(ok)) {
    drain(0, 1);
    return;
  }
  run_phase1(0);
  prep.advance();
  __syncthreads();

  for (int64_t q = 0; q < nseq; ++q) {
    const int64_t d0 = d0_of(cur);
    const int64_t d_ck = d0 + lg;  // training variant: the lane's channel
    if (cur.first()) {
      // a new piece: this lane's A values, and h from 0 or the predecessor's carry
      bool have = true;
      const bool cin_here = cur.carry_in();
      if (cin_here) {
        if (tid == 0) have = wait_carry(sched, w - 1);
        have = __syncthreads_and(have);  // also orders the carry reads after the wait
      }
      lane_load_decay<CF>(a, d0, lg, j, a2, ia);
      if (have && cin_here) {
        const float* cin = sched.carries + (int64_t)(w - 1) * CF::CH * CF::N;
        lane_load_state<CF>(h, [&](int cc) -> const float* {
          const int64_t i0 = ((int64_t)(w - 1) * CF::CH + lg * CPL + cc) * CF::N;
          return in_range(i0, CF::N, (int64_t)gridDim.x * CF::CH * CF::N) ? cin + (lg * CPL + cc) * CF::N
                                                                          : nullptr;
        }, j);
      } else {
        // a piece that starts the group (chunk 0) reads h0, if given
        lane_load_state<CF>(h, rows_in(const_cast<float*>(a.h0), cur.b, d0), j);
      }
      ok = ok && have;
    }
    run_phase2(h, a2, ia, ckpt_at(cur.b, d_ck, d_ck < a.dim, (int64_t)cur.c * CF::T));
    const bool cout_here = cur.carry_out();
    if (cout_here && writer) {
      float* cdst = sched.carries + (int64_t)w * CF::CH * CF::N;
      lane_store_state<CF>(h, [&](int cc) -> float* {
        const int64_t i0 = ((int64_t)w * CF::CH + lg * CPL + cc) * CF::N;
        return in_range(i0, CF::N, (int64_t)gridDim.x * CF::CH * CF::N) ? cdst + (lg * CPL + cc) * CF::N
                                                                       : nullptr;
      }, j);
      __threadfence();
    }
    if (cur.last() && writer) lane_store_state<CF>(h, rows_in(a.last_state, cur.b, d0), j);
    if (q + 1 < nseq) stage_in(q + 1, prep);
    if (!__syncthreads_and(ok)) {
      drain(q + 1, q + 1);
      return;
    }
    if (cout_here && tid == 0 && w != sched.skip_publish) publish_carry(sched, w);
    if (cur.g != D_g) {
      load_D(d0, D_it);
      D_g = cur.g;
    }
    const E* rc = reinterpret_cast<const E*>(raw(q));
    if (full_chunk(cur)) phase3<CF, true>(a, rc, sy, su, D_it, cur.b, d0, (int64_t)cur.c * CF::T, has_z);
    else phase3<CF, false>(a, rc, sy, su, D_it, cur.b, d0, (int64_t)cur.c * CF::T, has_z);
    if (q + 1 < nseq) {
      run_phase1(q + 1);
      prep.advance();
    }
    __syncthreads();
    if (tma && tid == 0 && q + 2 < nseq) {
      issue(q + 2);
      fetch.advance();
    }
    cur.advance();
  }
}

}  // namespace ssscan
