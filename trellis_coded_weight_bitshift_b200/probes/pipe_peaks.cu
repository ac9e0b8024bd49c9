// Per-SM issue/throughput probe for the instruction classes the trellis
// kernels are bound by: MUFU ex2/lg2, FFMA, FMNMX, packed FADD2, compare+select.
// Each thread runs 8 independent dependency chains; 4 CTAs of 256 threads per
// SM; results per SM per clock come from clock64 deltas, absolute rates from
// CUDA events.
#include <cstdio>
#include <cuda_runtime.h>
#define CH 8
template <int OP>
__global__ void probe(float *out, unsigned long long *cyc, int iters, float seed) {
  float x[CH];
  for (int c = 0; c < CH; ++c) x[c] = seed + threadIdx.x * 1e-3f + c;
  __syncthreads();
  const unsigned long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      if (OP == 0) { float y; asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x[c])); x[c] = y; }
      if (OP == 1) { float y; asm volatile("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x[c])); x[c] = y; }
      if (OP == 2) { x[c] = fmaf(x[c], 0.999f, 0.001f); }
      if (OP == 3) { x[c] = fminf(x[c], x[(c + 1) % CH] + 0.f); }
      if (OP == 4) {
        unsigned long long p, r;
        asm volatile("mov.b64 %0, {%1,%1};" : "=l"(p) : "f"(x[c]));
        asm volatile("add.rn.f32x2 %0, %1, %1;" : "=l"(r) : "l"(p));
        float lo, hi;
        asm volatile("mov.b64 {%0,%1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
        x[c] = lo;
      }
      if (OP == 5) { const bool p = x[c] < x[(c + 3) % CH]; x[c] = p ? x[c] * 1.0001f : x[c] + 1.f; }
    }
  }
  __syncthreads();
  const unsigned long long t1 = clock64();
  float acc = 0;
  for (int c = 0; c < CH; ++c) acc += x[c];
  out[blockIdx.x * blockDim.x + threadIdx.x] = acc;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <int OP>
static void run(const char *name, int sms) {
  const int blocks = sms * 4, threads = 256, iters = 4096;
  float *out;
  unsigned long long *cyc;
  cudaMalloc(&out, (size_t)blocks * threads * 4);
  cudaMalloc(&cyc, (size_t)blocks * 8);
  probe<OP><<<blocks, threads>>>(out, cyc, 16, 1.f);
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  cudaEventRecord(a);
  probe<OP><<<blocks, threads>>>(out, cyc, iters, 1.f);
  cudaEventRecord(b);
  cudaEventSynchronize(b);
  float ms;
  cudaEventElapsedTime(&ms, a, b);
  unsigned long long *h = new unsigned long long[blocks];
  cudaMemcpy(h, cyc, (size_t)blocks * 8, cudaMemcpyDeviceToHost);
  double mc = 0;
  for (int i = 0; i < blocks; ++i) mc = mc > h[i] ? mc : (double)h[i];
  const double ops = (double)blocks * threads * iters * CH;
  printf("%-10s results/s %.3e   per SM per clock %.1f   (clock implied %.0f MHz, %s)\n", name,
         ops / (ms * 1e-3), (ops / sms) / mc, mc / (ms * 1e-3) / 1e6,
         cudaGetErrorString(cudaGetLastError()));
  cudaFree(out);
  cudaFree(cyc);
  delete[] h;
}

int main() {
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  printf("SMs %d\n", sms);
  run<0>("ex2", sms);
  run<1>("lg2", sms);
  run<2>("ffma", sms);
  run<3>("fmnmx", sms);
  run<4>("fadd.f32x2", sms);
  run<5>("fsetp+sel", sms);
  return 0;
}
