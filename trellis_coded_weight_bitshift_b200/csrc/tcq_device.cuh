// Device-side building blocks shared by the trellis kernels (sm_100a).
//
//   * the 1MAD computed code [QTIP blog, "The codebook is computed"]: a 32-bit
//     LCG step, the byte sum of its output (one VABSDIFF4 against zero), the
//     centring by 510 and the scale 1/147.8;
//   * base-2 exponent/logarithm and reciprocal on the MUFU unit (PTX
//     ex2/lg2/rcp.approx);
//   * the shared-memory swizzle used by every state-vector exchange;
//   * small launch/validation helpers for the C ABI.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tcq.h"

namespace tcq {

constexpr uint32_t kLcgMul = 34038481u;
constexpr uint32_t kLcgAdd = 76625530u;

// Byte sum of the LCG output for state x (Irwin-Hall with n = 4).
__device__ __forceinline__ uint32_t one_mad_bytesum(uint32_t x) {
  return __vsadu4(x * kLcgMul + kLcgAdd, 0u);
}

// fp32 code value: the fp64 value (bytesum - 510) / 147.8 rounded once to
// fp32.  Used once per state at kernel start, so the exact fp64 division is
// affordable and the table is identical to the definition.
__device__ __forceinline__ float one_mad_f32(uint32_t x) {
  const double v = (double)((int)one_mad_bytesum(x) - 510) / 147.8;
  return __double2float_rn(v);
}

// fp32 value on the streaming decode path: (bytesum - 510) * RN(1/147.8).
// bytesum - 510 is formed exactly with the 2^23 magic-number trick; after the
// final round-to-nearest-even to fp16 this equals the fp16 rounding of the
// fp64 definition for all 1,021 byte sums (checked exhaustively by the tests).
__device__ __forceinline__ float one_mad_decode_f32(uint32_t x) {
  const uint32_t bs = one_mad_bytesum(x);
  const float centred = __fsub_rn(__uint_as_float(0x4B000000u | bs), 8389118.0f);
  return __fmul_rn(centred, 0x1.bb68f6p-8f);  // RN32(1/147.8)
}

// The same value for two states at once, arranged for throughput: the byte sum
// is a dot product with 0x01010101 whose accumulator carries the 2^23 exponent
// bits (IDP4A, integer multiply-add pipe), and the centring and scaling run as
// one packed fp32 pair (sub then mul, each correctly rounded per lane).
__device__ __forceinline__ unsigned long long one_mad_decode_f32x2(uint32_t x0, uint32_t x1) {
  const uint32_t m0 = __dp4a(x0 * kLcgMul + kLcgAdd, 0x01010101u, 0x4B000000u);
  const uint32_t m1 = __dp4a(x1 * kLcgMul + kLcgAdd, 0x01010101u, 0x4B000000u);
  unsigned long long v, c, r;
  asm("mov.b64 %0, {%1,%2};" : "=l"(v) : "r"(m0), "r"(m1));
  asm("mov.b64 %0, {%1,%1};" : "=l"(c) : "f"(8389118.0f));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(v), "l"(c));
  asm("mov.b64 %0, {%1,%1};" : "=l"(c) : "f"(0x1.bb68f6p-8f));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(r), "l"(c));
  return r;
}

// Packed fp32 pairs (sm_100a f32x2 arithmetic, round-to-nearest per lane).
// Each lane of sub/mul/add/fma.rn.f32x2 is the correctly rounded scalar
// operation.  Note: ptxas may fuse a packed mul whose only use is a packed add
// into one fma; code that needs the separately rounded product writes the
// square as fma(d, d, +0), which rounds exactly like d * d for d * d >= 0 and
// cannot be fused further.
typedef unsigned long long f2_t;
// Pair construction and halves in plain C++ (bit moves the compiler sees
// through, so a pair can live in two adjacent registers without copies).
__device__ __forceinline__ f2_t f2(float lo, float hi) {
  return ((f2_t)__float_as_uint(hi) << 32) | (f2_t)__float_as_uint(lo);
}
__device__ __forceinline__ float f2lo(f2_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2hi(f2_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ f2_t f2sub(f2_t a, f2_t b) {
  f2_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2_t f2mul(f2_t a, f2_t b) {
  f2_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2_t f2add(f2_t a, f2_t b) {
  f2_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2_t f2fma(f2_t a, f2_t b, f2_t c) {
  f2_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Reciprocal on the MUFU unit (PTX rcp.approx, a single special-function op).
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Tensor memory (sm_100a) as per-thread storage: a warp reaches the 32 TMEM
// lanes 32 (warp % 4) .. + 31, lane = its thread; an address is
// (lane << 16) | column, one column = one 32-bit word.  Allocation and
// release are warp-collective; every other call here is warp-collective too
// and touches only the calling thread's own lane.
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_dst, uint32_t ncols) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(d), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]), "=f"(r[7])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
               "%12, %13, %14, %15}, [%16];"
               : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]), "=f"(r[7]),
                 "=f"(r[8]), "=f"(r[9]), "=f"(r[10]), "=f"(r[11]), "=f"(r[12]), "=f"(r[13]), "=f"(r[14]),
                 "=f"(r[15])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
               "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
               "%30, %31}, [%32];"
               : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]), "=f"(r[7]),
                 "=f"(r[8]), "=f"(r[9]), "=f"(r[10]), "=f"(r[11]), "=f"(r[12]), "=f"(r[13]), "=f"(r[14]),
                 "=f"(r[15]), "=f"(r[16]), "=f"(r[17]), "=f"(r[18]), "=f"(r[19]), "=f"(r[20]), "=f"(r[21]),
                 "=f"(r[22]), "=f"(r[23]), "=f"(r[24]), "=f"(r[25]), "=f"(r[26]), "=f"(r[27]), "=f"(r[28]),
                 "=f"(r[29]), "=f"(r[30]), "=f"(r[31])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory swizzle of a state-vector index (float granularity).  Works on
// 16-byte units: unit u goes to u ^ ((u >> 3) & MASK).  It is a bijection, so
// any consistent use is correct; MASK = G/4 - 1 makes both the strided vector
// reads and the contiguous vector writes of a trellis step bank-conflict free.
template <int MASK>
__device__ __forceinline__ int swz(int idx) {
  const int u = idx >> 2;
  return (((u ^ ((u >> 3) & MASK))) << 2) | (idx & 3);
}

}  // namespace tcq

// Host-side helpers used by the C ABI translation units.
namespace tcq_host {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline tcq_status_t check_trellis(const tcq_trellis_t *tr) {
  if (!tr) return TCQ_ERR_INVALID_ARG;
  if (tr->L <= 0 || tr->k <= 0 || tr->V <= 0 || tr->seq_len <= 0) return TCQ_ERR_INVALID_ARG;
  if (tr->k != 2 || tr->V != 1) return TCQ_ERR_UNSUPPORTED;
  if (tr->L != 8 && tr->L != 12 && tr->L != 16) return TCQ_ERR_UNSUPPORTED;
  if (tr->seq_len > 256) return TCQ_ERR_UNSUPPORTED;
  return TCQ_OK;
}

inline tcq_status_t launch_status() {
  return cudaGetLastError() == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

inline int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

}  // namespace tcq_host
