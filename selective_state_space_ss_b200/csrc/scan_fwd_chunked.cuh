// scan_fwd_chunked.cuh -- channel-parallel fused selective-scan forward.
//
// One CTA owns CH consecutive channels d of one batch row b and walks the
// whole sequence in chunks of T timesteps.  Inside the CTA a warp holds
// 32/K channels; the K lanes of a channel each keep G = N/K of its states
// h[n] in fp32 registers for the whole sequence, so the state never touches
// memory (the SRAM-resident scan of "Mamba 深度解读报告", sec. 2.4, and the
// fused discretise/scan/readout kernel of "Mamba 选择性机制", sec. 3.2).
//
// Per chunk, with the inputs staged in shared memory by cp.async (double
// buffered, the next chunk's copy overlaps this chunk's math):
//   phase 1  per element: Delta = softplus(delta + bias), w = Delta * u,
//            and B, C widened to fp32 in a [t][state-group] layout;
//   phase 2  per (channel, state): A_bar = 2^(Delta * A * log2 e),
//            h = A_bar * h + w * B_t[n], partial readout sum_n C_t[n] h[n],
//            then a K-lane butterfly that leaves one timestep's full sum per
//            lane (B_t and C_t are read once per CTA and broadcast to every
//            channel, the per-token sharing of "从Transformer的痛点 ... Mamba",
//            sec. 4.2);
//   phase 3  per element: y = (s + D u) * SiLU(z), coalesced fp32 stores.
// The serial time loop inside a thread is the recurrence itself; the
// associative operator of "Mamba 选择性机制", sec. 3.1, is not needed here
// because no thread ever holds a time range whose carry-in is unknown.
#pragma once

#include "scan_common.cuh"

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
  int64_t batch, dim, seqlen;
  int softplus;
  int vec;  // 1: every row starts on a 16-byte boundary and 16-byte copies are used
};

template <typename Tin, int N_, int K_, int NWARPS_, int T_>
struct ChunkedCfg {
  using Elem = Tin;
  static constexpr int N = N_;            // states per channel
  static constexpr int K = K_;            // lanes per channel
  static constexpr int G = N / K;         // states per lane
  static constexpr int NWARPS = NWARPS_;
  static constexpr int T = T_;            // timesteps per chunk
  static constexpr int CPW = 32 / K;      // channels per warp
  static constexpr int CH = NWARPS * CPW; // channels per CTA
  static constexpr int NT = NWARPS * 32;
  static constexpr int VE = 16 / (int)sizeof(Tin);  // elements per 16-byte vector
  static constexpr int RS = T + VE;                  // staged row stride (elements)
  static constexpr int RAW_ROWS = 3 * CH + 2 * N;    // u, delta, z rows then B, C rows
  static constexpr int RAW_BYTES = RAW_ROWS * RS * (int)sizeof(Tin);
  static constexpr int DW_STRIDE = CH + 1;           // float4 per half-row (pads banks)
  static constexpr int DW_BYTES = (T / 2) * DW_STRIDE * 16;
  static constexpr int BC_STRIDE = 2 * N + 4;        // floats per timestep
  static constexpr int BC_BYTES = T * BC_STRIDE * 4;
  static constexpr int SY_STRIDE = T + 4;            // floats per channel row
  static constexpr int SY_BYTES = CH * SY_STRIDE * 4;
  static constexpr int SMEM_BYTES = 2 * RAW_BYTES + DW_BYTES + BC_BYTES + SY_BYTES;

  static_assert(N % K == 0 && 32 % K == 0, "lane split");
  static_assert(T % 32 == 0, "chunk length");
  static_assert(G == 1 || G % 2 == 0, "state group");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// ---------------------------------------------------------------- loads ---

template <class CF>
__device__ __forceinline__ void load_chunk(const FwdArgs& a, typename CF::Elem* raw,
                                           int64_t b, int64_t d0, int64_t t0) {
  using E = typename CF::Elem;
  const int tid = threadIdx.x;
  const int64_t L = a.seqlen, D = a.dim;
  const E* srcs[5] = {static_cast<const E*>(a.u), static_cast<const E*>(a.delta),
                      static_cast<const E*>(a.z), static_cast<const E*>(a.B),
                      static_cast<const E*>(a.C)};
  if (a.vec) {
    constexpr int VPR = CF::T / CF::VE;
    for (int i = tid; i < CF::RAW_ROWS * VPR; i += CF::NT) {
      const int r = i / VPR, v = i - r * VPR;
      const int64_t t = t0 + (int64_t)v * CF::VE;
      E* dst = raw + r * CF::RS + v * CF::VE;
      const E* src = nullptr;
      if (t < L) {
        if (r < 3 * CF::CH) {
          const int which = r / CF::CH, c = r - which * CF::CH;
          const int64_t d = d0 + c;
          if (d < D && srcs[which]) src = srcs[which] + ((b * D + d) * L + t);
        } else {
          const int rr = r - 3 * CF::CH, which = rr / CF::N, n = rr - which * CF::N;
          src = srcs[3 + which] + ((b * CF::N + n) * L + t);
        }
      }
      if (src) cp_async16(dst, src);
      else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
  } else {
    for (int i = tid; i < CF::RAW_ROWS * CF::T; i += CF::NT) {
      const int r = i / CF::T, tt = i - r * CF::T;
      const int64_t t = t0 + tt;
      E val = zero_elem<E>();
      if (t < L) {
        if (r < 3 * CF::CH) {
          const int which = r / CF::CH, c = r - which * CF::CH;
          const int64_t d = d0 + c;
          if (d < D && srcs[which]) val = srcs[which][(b * D + d) * L + t];
        } else {
          const int rr = r - 3 * CF::CH, which = rr / CF::N, n = rr - which * CF::N;
          val = srcs[3 + which][(b * CF::N + n) * L + t];
        }
      }
      raw[r * CF::RS + tt] = val;
    }
  }
}

// ------------------------------------------------------------- phase 1 ---

template <class CF>
__device__ __forceinline__ void phase1(const FwdArgs& a, const typename CF::Elem* raw,
                                       float4* dw, float* bc, const float* s_bias,
                                       int64_t d0, int64_t t0) {
  const int tid = threadIdx.x;
  constexpr int QPR = CF::T / 4;
  const int64_t L = a.seqlen;
  for (int i = tid; i < CF::CH * QPR; i += CF::NT) {
    const int c = i / QPR, q = i - c * QPR;
    const float4 dl = load4_f32(raw + (CF::CH + c) * CF::RS + 4 * q);
    const float4 uu = load4_f32(raw + c * CF::RS + 4 * q);
    const float bias = s_bias[c];
    const bool chan_ok = d0 + c < a.dim;
    float dv[4] = {dl.x, dl.y, dl.z, dl.w};
    float uv[4] = {uu.x, uu.y, uu.z, uu.w};
    float delt[4], w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool ok = chan_ok && (t0 + 4 * q + k < L);
      float x = dv[k] + bias;
      x = a.softplus ? softplus_f32(x) : x;
      delt[k] = ok ? x : 0.f;  // padding steps: A_bar = 1, B_bar u = 0 (state unchanged)
      w[k] = delt[k] * uv[k];
    }
    dw[(2 * q) * CF::DW_STRIDE + c] = make_float4(delt[0], w[0], delt[1], w[1]);
    dw[(2 * q + 1) * CF::DW_STRIDE + c] = make_float4(delt[2], w[2], delt[3], w[3]);
  }
  // B and C: [n][t] staged rows -> [t][group j][B (G values), C (G values)]
  for (int i = tid; i < 2 * CF::N * QPR; i += CF::NT) {
    const int r = i / QPR, q = i - r * QPR;
    const int which = r / CF::N, n = r - which * CF::N;
    const float4 v = load4_f32(raw + (3 * CF::CH + r) * CF::RS + 4 * q);
    const int j = n / CF::G, g = n - j * CF::G;
    float* col = bc + (4 * q) * CF::BC_STRIDE + j * 2 * CF::G + which * CF::G + g;
    col[0] = v.x;
    col[CF::BC_STRIDE] = v.y;
    col[2 * CF::BC_STRIDE] = v.z;
    col[3 * CF::BC_STRIDE] = v.w;
  }
}

// ------------------------------------------------------------- phase 2 ---

// Sum the four per-lane partial readouts over the K lanes of a channel and
// store the full sums for timesteps t..t+3 into the channel's sy row.
template <int K>
__device__ __forceinline__ void reduce_store4(float s0, float s1, float s2, float s3,
                                              float* sy_t, int j) {
  if constexpr (K == 1) {
    *reinterpret_cast<float4*>(sy_t) = make_float4(s0, s1, s2, s3);
  } else if constexpr (K == 2) {
    const bool hi = j & 1;
    float k0 = hi ? s2 : s0, k1 = hi ? s3 : s1;
    const float o0 = hi ? s0 : s2, o1 = hi ? s1 : s3;
    k0 += __shfl_xor_sync(kFullMask, o0, 1);
    k1 += __shfl_xor_sync(kFullMask, o1, 1);
    *reinterpret_cast<float2*>(sy_t + 2 * j) = make_float2(k0, k1);
  } else {
#pragma unroll
    for (int m = K / 2; m >= 4; m /= 2) {
      s0 += __shfl_xor_sync(kFullMask, s0, m);
      s1 += __shfl_xor_sync(kFullMask, s1, m);
      s2 += __shfl_xor_sync(kFullMask, s2, m);
      s3 += __shfl_xor_sync(kFullMask, s3, m);
    }
    const bool b1 = j & 2;
    float k0 = b1 ? s2 : s0, k1 = b1 ? s3 : s1;
    const float o0 = b1 ? s0 : s2, o1 = b1 ? s1 : s3;
    k0 += __shfl_xor_sync(kFullMask, o0, 2);
    k1 += __shfl_xor_sync(kFullMask, o1, 2);
    const bool b0 = j & 1;
    float kk = b0 ? k1 : k0;
    const float oo = b0 ? k0 : k1;
    kk += __shfl_xor_sync(kFullMask, oo, 1);
    if (j < 4) sy_t[j] = kk;
  }
}

template <class CF>
__device__ __forceinline__ void phase2(const float4* dw, const float* bc, float* sy,
                                       float (&h)[CF::G], const float (&a2)[CF::G],
                                       int c, int j) {
  constexpr int G = CF::G;
  const float* bcj = bc + j * 2 * G;
  float* syc = sy + c * CF::SY_STRIDE;
#pragma unroll 1
  for (int t = 0; t < CF::T; t += 4) {
    float s[4];
#pragma unroll
    for (int k2 = 0; k2 < 4; k2 += 2) {
      const float4 p = dw[((t + k2) >> 1) * CF::DW_STRIDE + c];
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const float dl = kk ? p.z : p.x;
        const float w = kk ? p.w : p.y;
        const float* row = bcj + (t + k2 + kk) * CF::BC_STRIDE;
        float Bv[G], Cv[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int g = 0; g < G; g += 4) {
            const float4 bq = *reinterpret_cast<const float4*>(row + g);
            const float4 cq = *reinterpret_cast<const float4*>(row + G + g);
            Bv[g] = bq.x; Bv[g + 1] = bq.y; Bv[g + 2] = bq.z; Bv[g + 3] = bq.w;
            Cv[g] = cq.x; Cv[g + 1] = cq.y; Cv[g + 2] = cq.z; Cv[g + 3] = cq.w;
          }
        } else {
#pragma unroll
          for (int g = 0; g < G; ++g) { Bv[g] = row[g]; Cv[g] = row[G + g]; }
        }
        float acc = 0.f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float abar = ex2_approx(dl * a2[g]);
          h[g] = fmaf(abar, h[g], w * Bv[g]);
          acc = fmaf(Cv[g], h[g], acc);
        }
        s[k2 + kk] = acc;
      }
    }
    reduce_store4<CF::K>(s[0], s[1], s[2], s[3], syc + t, j);
  }
}

// ------------------------------------------------------------- phase 3 ---

template <class CF>
__device__ __forceinline__ void phase3(const FwdArgs& a, const typename CF::Elem* raw,
                                       const float* sy, const float* s_D,
                                       int64_t b, int64_t d0, int64_t t0, bool has_z) {
  const int tid = threadIdx.x;
  constexpr int QPR = CF::T / 4;
  const int64_t L = a.seqlen, D = a.dim;
  for (int i = tid; i < CF::CH * QPR; i += CF::NT) {
    const int c = i / QPR, q = i - c * QPR;
    const int64_t d = d0 + c, t = t0 + 4 * q;
    if (d >= D || t >= L) continue;
    const float4 s = *reinterpret_cast<const float4*>(sy + c * CF::SY_STRIDE + 4 * q);
    const float4 uu = load4_f32(raw + c * CF::RS + 4 * q);
    const float Dd = s_D[c];
    float y[4] = {fmaf(Dd, uu.x, s.x), fmaf(Dd, uu.y, s.y), fmaf(Dd, uu.z, s.z), fmaf(Dd, uu.w, s.w)};
    if (has_z) {
      const float4 zz = load4_f32(raw + (2 * CF::CH + c) * CF::RS + 4 * q);
      y[0] *= silu_f32(zz.x);
      y[1] *= silu_f32(zz.y);
      y[2] *= silu_f32(zz.z);
      y[3] *= silu_f32(zz.w);
    }
    float* dst = a.y + (b * D + d) * L + t;
    if (a.vec && t + 3 < L) {
      *reinterpret_cast<float4*>(dst) = make_float4(y[0], y[1], y[2], y[3]);
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (t + k < L) dst[k] = y[k];
    }
  }
}

// -------------------------------------------------------------- kernel ---

template <class CF>
__global__ void __launch_bounds__(CF::NT) scan_fwd_chunked_kernel(FwdArgs a) {
  using E = typename CF::Elem;
  extern __shared__ __align__(16) unsigned char smem[];
  E* raw0 = reinterpret_cast<E*>(smem);
  E* raw1 = reinterpret_cast<E*>(smem + CF::RAW_BYTES);
  float4* dw = reinterpret_cast<float4*>(smem + 2 * CF::RAW_BYTES);
  float* bc = reinterpret_cast<float*>(smem + 2 * CF::RAW_BYTES + CF::DW_BYTES);
  float* sy = reinterpret_cast<float*>(smem + 2 * CF::RAW_BYTES + CF::DW_BYTES + CF::BC_BYTES);
  __shared__ float s_bias[CF::CH], s_D[CF::CH];

  const int64_t tiles_per_b = (a.dim + CF::CH - 1) / CF::CH;
  const int64_t b = blockIdx.x / tiles_per_b;
  const int64_t d0 = (blockIdx.x - b * tiles_per_b) * CF::CH;
  const int64_t L = a.seqlen;
  const bool has_z = a.z != nullptr;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = warp * CF::CPW + lane / CF::K;  // this lane's channel within the CTA
  const int j = lane % CF::K;                   // this lane's state group
  const int64_t d = d0 + c;
  const bool chan_ok = d < a.dim;

  for (int i = tid; i < CF::CH; i += CF::NT) {
    const int64_t dd = d0 + i;
    s_bias[i] = (dd < a.dim && a.delta_bias) ? a.delta_bias[dd] : 0.f;
    s_D[i] = (dd < a.dim && a.D) ? a.D[dd] : 0.f;
  }

  float h[CF::G], a2[CF::G];
#pragma unroll
  for (int g = 0; g < CF::G; ++g) {
    h[g] = 0.f;
    a2[g] = chan_ok ? a.A[d * CF::N + j * CF::G + g] * 1.4426950408889634f : 0.f;
  }

  const int64_t nchunks = (L + CF::T - 1) / CF::T;
  load_chunk<CF>(a, raw0, b, d0, 0);
  if (nchunks > 1) load_chunk<CF>(a, raw1, b, d0, CF::T);
  // wait for chunk 0 only: chunk 1's group may stay in flight
  if (a.vec) {
    if (nchunks > 1) asm volatile("cp.async.wait_group 1;\n" ::: "memory");
    else cp_async_wait_all();
  }
  __syncthreads();
  phase1<CF>(a, raw0, dw, bc, s_bias, d0, 0);
  __syncthreads();

  for (int64_t k = 0; k < nchunks; ++k) {
    E* cur = (k & 1) ? raw1 : raw0;
    E* nxt = (k & 1) ? raw0 : raw1;
    phase2<CF>(dw, bc, sy, h, a2, c, j);
    if (a.vec) cp_async_wait_all();  // chunk k+1 has landed
    __syncthreads();
    phase3<CF>(a, cur, sy, s_D, b, d0, k * CF::T, has_z);
    if (k + 1 < nchunks) phase1<CF>(a, nxt, dw, bc, s_bias, d0, (k + 1) * CF::T);
    __syncthreads();
    if (k + 2 < nchunks) load_chunk<CF>(a, cur, b, d0, (k + 2) * CF::T);
  }

  if (a.last_state && chan_ok) {
    float* dst = a.last_state + ((b * a.dim + d) * CF::N + j * CF::G);
#pragma unroll
    for (int g = 0; g < CF::G; ++g) dst[g] = h[g];
  }
}

}  // namespace ssscan
