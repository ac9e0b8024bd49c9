// Write-stream bandwidth of this GPU: 1 GiB written with 16-byte vector
// stores (default and evict-first policy) and with bulk shared->global copies
// (cp.async.bulk, 16 KiB per copy, four in flight per CTA).  Best of 10 by
// CUDA events.
#include <cstdint>
#include <cstdio>

__global__ void store_v4(float4 *p, size_t n) {
  const float4 v = make_float4(1.f, 2.f, 3.f, 4.f);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    p[i] = v;
}

__global__ void store_v4_cs(float4 *p, size_t n) {
  const float4 v = make_float4(1.f, 2.f, 3.f, 4.f);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    __stcs(p + i, v);
}

constexpr int kChunk = 16384;

__global__ void store_bulk(char *p, size_t nbytes) {
  extern __shared__ __align__(128) float4 buf[];
  for (int i = threadIdx.x; i < kChunk / 16; i += blockDim.x) buf[i] = make_float4(1.f, 2.f, 3.f, 4.f);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t src = (uint32_t)__cvta_generic_to_shared(buf);
    for (size_t c = blockIdx.x; c < nbytes / kChunk; c += gridDim.x) {
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(p + c * kChunk),
                   "r"(src), "r"(kChunk)
                   : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 4;" ::: "memory");
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
}

int main() {
  const size_t bytes = 1ull << 30;
  char *p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return 1;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  cudaFuncSetAttribute(store_bulk, cudaFuncAttributeMaxDynamicSharedMemorySize, kChunk);
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  const char *names[] = {"16-byte stores", "16-byte stores, evict-first", "bulk copies from shared memory"};
  for (int k = 0; k < 3; ++k) {
    float best = 1e30f;
    for (int rep = 0; rep < 11; ++rep) {
      cudaEventRecord(a);
      if (k == 0) store_v4<<<sms * 8, 256>>>(reinterpret_cast<float4 *>(p), bytes / 16);
      if (k == 1) store_v4_cs<<<sms * 8, 256>>>(reinterpret_cast<float4 *>(p), bytes / 16);
      if (k == 2) store_bulk<<<sms * 4, 32, kChunk>>>(p, bytes);
      cudaEventRecord(b);
      if (cudaDeviceSynchronize() != cudaSuccess) return 2;
      float ms = 0.f;
      cudaEventElapsedTime(&ms, a, b);
      if (rep > 0 && ms < best) best = ms;
    }
    printf("write of 1024 MiB, %s: %.1f GB/s\n", names[k], bytes / (best * 1e6));
  }
  cudaFree(p);
  return 0;
}
