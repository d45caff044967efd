// probe_rates.cu -- issue-rate probe for the units the scan is bound by:
// the special-function unit (ex2.approx.ftz.f32), the FMA pipe (fma.rn.f32)
// and packed fp32x2 FMA (fma.rn.f32x2).  Independent chains per thread, all
// CTAs resident (148 x 4 CTAs x 192 threads); cycles from clock64.  Every
// thread writes one float of a buffer sized grid x block.
//   build: python -m selective_state_space_ss_b200.build (writes probe_rates)
//   run:   selective_state_space_ss_b200/probe_rates
#include <cstdio>
#include <cuda_runtime.h>

__device__ __forceinline__ float ex2(float x) { float y; asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x)); return y; }

template <int CH>
__global__ void ex2_tput(float* out, int iters, long long* cyc) {
  float a[CH];
#pragma unroll
  for (int c = 0; c < CH; ++c) a[c] = 0.001f * (threadIdx.x + c);
  long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < CH; ++c) a[c] = ex2(-a[c]);
  }
  long long t1 = clock64();
  float s = 0;
#pragma unroll
  for (int c = 0; c < CH; ++c) s += a[c];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <int CH>
__global__ void ffma_tput(float* out, int iters, long long* cyc) {
  float a[CH];
#pragma unroll
  for (int c = 0; c < CH; ++c) a[c] = 0.001f * (threadIdx.x + c);
  long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < CH; ++c) a[c] = fmaf(a[c], 0.999f, 0.0001f);
  }
  long long t1 = clock64();
  float s = 0;
#pragma unroll
  for (int c = 0; c < CH; ++c) s += a[c];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <int CH>
__global__ void ffma2_tput(float* out, int iters, long long* cyc) {
  unsigned long long a[CH];
  const float m = 0.999f, ad = 0.0001f;
  unsigned long long mm, aa;
  asm("mov.b64 %0, {%1, %2};" : "=l"(mm) : "f"(m), "f"(m));
  asm("mov.b64 %0, {%1, %2};" : "=l"(aa) : "f"(ad), "f"(ad));
#pragma unroll
  for (int c = 0; c < CH; ++c) { float x = 0.001f * (threadIdx.x + c); asm("mov.b64 %0, {%1, %2};" : "=l"(a[c]) : "f"(x), "f"(x)); }
  long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < CH; ++c) asm volatile("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(a[c]) : "l"(mm), "l"(aa));
  }
  long long t1 = clock64();
  float s = 0;
#pragma unroll
  for (int c = 0; c < CH; ++c) { float lo, hi; asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a[c])); s += lo + hi; }
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <class K>
void run(const char* name, K kern, int chains, double ops_per_iter_chain) {
  int sms = 148, bpsm = 4, threads = 192, iters = 4096;
  int blocks = sms * bpsm;
  float* out; long long* cyc;
  cudaMalloc(&out, sizeof(float) * blocks * threads);
  cudaMalloc(&cyc, sizeof(long long) * blocks);
  kern<<<blocks, threads>>>(out, 64, cyc);
  cudaEvent_t e0, e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
  cudaEventRecord(e0);
  kern<<<blocks, threads>>>(out, iters, cyc);
  cudaEventRecord(e1);
  cudaEventSynchronize(e1);
  float ms; cudaEventElapsedTime(&ms, e0, e1);
  long long* hc = new long long[blocks];
  cudaMemcpy(hc, cyc, sizeof(long long) * blocks, cudaMemcpyDeviceToHost);
  double maxc = 0, sumc = 0; for (int i = 0; i < blocks; ++i) { maxc = hc[i] > maxc ? hc[i] : maxc; sumc += hc[i]; }
  double total = (double)blocks * threads * iters * chains * ops_per_iter_chain;
  double per_sm_per_clk = total / sms / maxc;
  printf("%-12s chains=%2d  %.3f ms  %.1f Gop/s  %.2f op/clk/SM (max cyc %.0f, avg %.0f)  implied clock %.0f MHz\n",
         name, chains, ms, total / ms / 1e6, per_sm_per_clk, maxc, sumc / blocks, maxc / (ms * 1e3));
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) printf("error: %s\n", cudaGetErrorString(err));
  delete[] hc; cudaFree(out); cudaFree(cyc);
}

int main() {
  run("ex2", ex2_tput<8>, 8, 1);
  run("ex2", ex2_tput<16>, 16, 1);
  run("ffma", ffma_tput<8>, 8, 1);
  run("ffma", ffma_tput<16>, 16, 1);
  run("ffma2", ffma2_tput<8>, 8, 2);
  run("ffma2", ffma2_tput<16>, 16, 2);
  return 0;
}
