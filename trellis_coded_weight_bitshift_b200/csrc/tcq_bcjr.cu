// BCJR forward-backward on the bitshift trellis at temperature temp, and the
// vector-Jacobian product of the soft codeword.
//
// [BCJR-QAT abstract] the Viterbi argmax is replaced by the forward-backward
// sum-product recursion at temperature temp; the soft codeword is the
// Boltzmann expectation of the code over trellis walks and is exactly
// differentiable.  With E(x) = sum_t (code(x_t) - s_t)^2 and p(x) ~ exp(-E/temp)
// (free start, free end):
//   alpha_0(j) = -e_0(j)/temp,  alpha_t(j) = LSE_a alpha_{t-1}(pred_a j) - e_t(j)/temp
//   beta_{T-1} = 0,             beta_t(i)  = LSE_b [beta_{t+1}(succ_b i) - e_{t+1}(succ_b i)/temp]
//   soft_t = sum_j softmax_j(alpha_t + beta_t) code_j
// Everything here runs in base 2 (kappa = log2(e)/temp scales the energy) on
// the MUFU ex2/lg2 units, fp32.  Each step's emission is taken relative to r,
// the target clamped to the code range: -kappa (c - s)^2 differs from
// d (-kappa d + 2 kappa (s - r)), d = c - r, by a constant of the step, which
// cancels in every expectation and is added back to log Z in fp64; for a
// target outside the range the states that compete then carry small,
// accurately rounded emissions.
//
// Structure (k = 2, the same one as the Viterbi kernel):
//   * forward: the four states j = 4q + b share one log-sum-exp over their
//     predecessors, A_t(q) = LSE_a alpha_{t-1}(q | a << (L-2)), so the state
//     vector carried between steps is A (2^(L-2) values) and
//     alpha_t(p) = A_t(p >> 2) - kappa e_t(p) is rebuilt on the fly;
//   * backward: beta_t(i) depends only on i's low L-2 bits,
//     B_t(r) = LSE_b [B_{t+1}((4r + b) mod 2^(L-2)) - kappa e_{t+1}(4r + b)],
//     and thread w evaluates exactly the groups r whose states 4r + b are its
//     forward predecessor states, so the code values in its registers serve
//     both passes (the backward reads G contiguous values, writes four runs:
//     the mirror image of the forward step);
//   * combine: alpha_{t+1}(4r+b) + beta_{t+1}(4r+b) = A_{t+1}(r) + y_b where
//     y_b are the four inputs of the backward log-sum-exp for r, so the soft
//     codeword reuses those four exponentials: taken against the combine's
//     exponent reference K they are the posteriors themselves (L = 12, 16),
//     or, relative to their maximum, they take one more for the group weight
//     (L = 8);
//   * A_t is renormalised every step by the running maximum (a constant per
//     step, global over the sequence), and so is B; the constants are tracked
//     to place the combine's exponent reference K_t = log2 Z - (constants)
//     near zero, and soft_t = num_t / den_t cancels K_t exactly;
//   * the forward spills, per thread and per step, the A values it read to
//     its private slice of the workspace, and the backward reads them back in
//     reverse order (thread-private, so no inter-thread ordering is needed).
//
// Gradient (GRAD = true): d soft_t / d s_u = (2/temp) Cov(code(x_t), code(x_u)),
// so grad_u = (2/temp) Cov(F, code(x_u)) with F = sum_t v_t (code(x_t) - soft_t)
// (centred by the forward soft codeword when it is given, else by the target
// clamped to the code range: any per-step constant leaves the covariance
// unchanged, and a centre near the codes keeps F small).  E[F | x_u = j]
// splits by the Markov property into a prefix part phi (forward expectation
// recursion, weights = the forward softmax over predecessors) and a suffix
// part psi (backward recursion, weights = the backward softmax over
// successors); both reuse the exponentials of the log-sum-exps above.
#include <algorithm>
#include <mutex>

#include "tcq_device.cuh"

namespace tcq {

// Cache prefetch of a global address (no register result).
template <int LEVEL>
__device__ __forceinline__ void prefetch_global(const void *p) {
  if constexpr (LEVEL == 1) asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
  else if constexpr (LEVEL == 2) asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

#ifndef TCQ_SPILL_PREFETCH_LEVEL
#define TCQ_SPILL_PREFETCH_LEVEL 2
#endif

// log2(2^x0 + 2^x1 + 2^x2 + 2^x3) with three ex2: after a min/max network
// the largest term is exactly 1.
__device__ __forceinline__ float lse4_base2(float x0, float x1, float x2, float x3) {
  const float hi01 = fmaxf(x0, x1), lo01 = fminf(x0, x1);
  const float hi23 = fmaxf(x2, x3), lo23 = fminf(x2, x3);
  const float mx = fmaxf(hi01, hi23), mo = fminf(hi01, hi23);
  const float S = (1.0f + ex2(lo01 - mx)) + (ex2(lo23 - mx) + ex2(mo - mx));
  return mx + lg2(S);
}

template <int L_, int G_, int SPC_, int AREG_, int NBUF_, bool GRAD_, int MINB_ = 1,
          bool TMEMC_ = false, bool MSG2_ = false>
struct BcjrCfg {
  static constexpr int L = L_, G = G_, SPC = SPC_, AREG = AREG_, NBUF = NBUF_;
  static constexpr int MINB = MINB_;                // CTAs per SM the registers must allow
  static constexpr bool GRAD = GRAD_;
  static constexpr int NG = 1 << (L - 2);
  static constexpr int TPS = NG / G;
  static constexpr int NT = TPS * SPC;
  static constexpr int GQ = G / 4;
  static constexpr int ASM = 4 - AREG;
  static constexpr int HREG = AREG / 2, HS = 2 - HREG;          // digit pairs: registers | elsewhere
  // the HS pairs not in registers sit in tensor memory (TMEMC) or shared memory
  static constexpr bool TMEMC = TMEMC_;
  static constexpr int TCPT = TMEMC ? HS * G * 2 : 0;              // TMEM columns per thread
  static constexpr int TCOLS = TCPT * (NT / 128) <= 32 ? 32 : TCPT * (NT / 128);  // per CTA
  static constexpr int NPART = TPS >= 32 ? TPS / 32 : 1;       // partial records per sequence
  // several warp-aligned sequences in one CTA step independently, each on its
  // own named barrier; they share one copy of the code values
  static constexpr bool NAMED = SPC > 1 && TPS % 32 == 0;
  // several sequences per warp (L = 8: 16 threads each): a sequence steps on
  // a warp barrier, since its threads exchange values only with each other
  static constexpr bool WARPSEQ = SPC > 1 && TPS < 32 && 32 % TPS == 0;
  // backward exponents against the combine's reference, so that the four
  // successor terms are posteriors (one ex2 and a maximum fewer per group);
  // it puts the spilled A on the B recursion's path, which the L = 8
  // gradient (its spill read inside the step) cannot hide; the soft passes
  // read it from registers loaded a step ahead (L = 8 soft with the spill
  // read in the step: 0.158 -> 0.171 ms on 64 sequences; L = 12 and 16 gain
  // 1-3% soft and 3% soft + VJP)
  static constexpr bool POSTB = !WARPSEQ || !GRAD;
  static constexpr int PREC = 8;                                 // floats per partial record
  static constexpr int SWZ = (GQ >= 8 ? 7 : GQ - 1);
  static constexpr int NV = GRAD ? 2 : 1;                        // carried vectors (A | A, Phi)
  static constexpr int SPILL = NV * G;                           // floats spilled per thread-step
  // MSG2 (gradient, NBUF = 1): the message vector (A, B) is double-buffered and
  // read block by block after the step's first barrier; only the expectation
  // vector (Phi, Psi) is single-buffered and read ahead of it
  static constexpr bool MSG2 = MSG2_;
  static constexpr int VPS = MSG2 ? 3 : NBUF * NV;              // state vectors per sequence
  static constexpr size_t smem_floats() {
    return (size_t)SPC * VPS * NG                                  // state vectors
           + (TMEMC ? 0 : (size_t)ASM * G * TPS)                    // smem code values
           + (size_t)SPC * 256 * (GRAD ? 4 : 2)                     // s, kappa*D (+ v, soft)
           + (size_t)SPC * 256                                       // CA_t increments
           + (size_t)2 * SPC * NPART * PREC;                        // partial records
  }
  static constexpr size_t smem_bytes() { return smem_floats() * sizeof(float); }
  // Steps are finished after the backward: the per-step sums go to the
  // workspace and the sequence's threads turn them into outputs in parallel
  // (finishing each step on one thread during the sweep stalls the other warps
  // of the sequence at the next barrier).
  static constexpr int NQS = GRAD ? 4 : 2;                        // sums per record
  // per resident sequence: the spilled messages, then the per-step partial
  // sums (numerator, denominator; gradient: and the two moments) of each
  // warp; a whole number of 256-byte units, so that every slot (read as
  // float4) stays 16-byte aligned
  __host__ __device__ static constexpr size_t ws_floats_per_slot(int T) {
    return ((size_t)T * NV * NG + (size_t)T * NPART * NQS + 63) / 64 * 64;
  }
  static_assert(NG % G == 0 && G % 4 == 0, "bad split");
  static_assert(AREG % 2 == 0, "code values are held in digit pairs");
  static_assert(!TMEMC || (SPC == 1 && NT % 128 == 0 && (TCOLS & (TCOLS - 1)) == 0 && TCOLS <= 512 &&
                           G % 8 == 0), "tensor-memory code layout");
  static_assert(SPILL % 4 == 0, "spill in float4 chunks");
  static_assert(!MSG2 || (GRAD && NBUF == 1 && GQ % 4 == 0), "split buffering is for the gradient");
  static_assert(!NAMED || (SPC <= 15 && !TMEMC), "named barriers 1..15, code values in shared memory");
  static_assert(!WARPSEQ || !TMEMC, "warp-stepped sequences keep their code values in shared memory");
};

// Barrier over the threads of one sequence: named barrier 1 + ls when the CTA
// holds several warp-aligned sequences, the warp barrier when a warp holds
// whole sequences, else the CTA barrier.
template <class C>
__device__ __forceinline__ void seq_sync(int ls) {
  if constexpr (C::NAMED) asm volatile("bar.sync %0, %1;" ::"r"(1 + ls), "n"(C::TPS) : "memory");
  else if constexpr (C::WARPSEQ) __syncwarp();
  else __syncthreads();
}

// Code values are held as vertical pairs over the predecessor digit:
// pair (h, i) = (code of state 2h NG + G w + i, code of state (2h+1) NG + G w + i).
// Digit pairs h < HREG live in registers; the others in tensor memory (this
// thread's lane, columns col0 + 2 ((h - HREG) G + i) and + 1) or in shared
// memory as float2 [HS][G][TPS] (consecutive lanes read consecutive pairs).
template <class C>
using CodeRegs = f2_t[C::HREG > 0 ? C::HREG : 1][C::G];

template <class C>
struct CodeSrc {
  const CodeRegs<C> &cv;
  const float2 *Csm;
  uint32_t taddr;                                          // this thread's TMEM lane, column 0
  int w;
  // N consecutive pairs (h, i0 .. i0 + N - 1); N = 4, 8 or 16, i0 a multiple of N
  template <int N>
  __device__ __forceinline__ void pairs(int h, int i0, f2_t (&out)[N]) const {
    if (h < C::HREG) {
#pragma unroll
      for (int n = 0; n < N; ++n) out[n] = cv[h < C::HREG ? h : 0][i0 + n];
    } else if constexpr (C::TMEMC) {
      float r[2 * N];
      const uint32_t col = 2 * ((h - C::HREG) * C::G + i0);
      if constexpr (N == 4) tmem_ld8(taddr + col, r);
      else if constexpr (N == 8) tmem_ld16(taddr + col, r);
      else tmem_ld32(taddr + col, r);
      tmem_wait_ld();
#pragma unroll
      for (int n = 0; n < N; ++n) out[n] = f2(r[2 * n], r[2 * n + 1]);
    } else {
#pragma unroll
      for (int n = 0; n < N; ++n) {
        const float2 v = Csm[((h - C::HREG) * C::G + i0 + n) * C::TPS + w];
        out[n] = f2(v.x, v.y);
      }
    }
  }
  // pairs (0, i0 ..) and (1, i0 ..) of 4 consecutive indices, with a single
  // tensor-memory wait when both come from there
  __device__ __forceinline__ void both_pairs4(int i0, f2_t (&out0)[4], f2_t (&out1)[4]) const {
    if constexpr (C::TMEMC && C::HREG == 0) {
      float r0[8], r1[8];
      tmem_ld8(taddr + 2 * i0, r0);
      tmem_ld8(taddr + 2 * (C::G + i0), r1);
      tmem_wait_ld();
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        out0[n] = f2(r0[2 * n], r0[2 * n + 1]);
        out1[n] = f2(r1[2 * n], r1[2 * n + 1]);
      }
    } else {
      pairs<4>(0, i0, out0);
      pairs<4>(1, i0, out1);
    }
  }
};

// Reduce within the TPS lanes of a sequence (TPS < 32) or the whole warp.
template <int TPS, class Op>
__device__ __forceinline__ float lane_reduce(float v, Op op) {
  constexpr int WL = TPS < 32 ? TPS : 32;
#pragma unroll
  for (int off = WL / 2; off > 0; off >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

struct MaxOp { __device__ float operator()(float a, float b) const { return fmaxf(a, b); } };

// Maximum over the TPS lanes of a sequence: one warp-wide redux when the
// sequence spans whole warps, else a shuffle tree.
template <int TPS>
__device__ __forceinline__ float seq_max(float v) {
  if constexpr (TPS >= 32) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
  } else {
    return lane_reduce<TPS>(v, MaxOp());
  }
}

// Sums of NQ (2 or 4) values over the WL = min(TPS, 32) lanes of a sequence
// in one shuffle tree: the first levels exchange different quantities, so the
// lane at offset o (within the WL lanes) ends with the full sum of quantity
// o / (WL / NQ).
template <int TPS, int NQ>
__device__ __forceinline__ float seq_sums(const float (&v)[NQ], int lane) {
  constexpr int WL = TPS < 32 ? TPS : 32;
  static_assert(NQ == 2 || NQ == 4, "two or four quantities");
  float y;
  if constexpr (NQ == 4) {
    const bool h1 = lane & (WL / 2);
    float k0 = h1 ? v[2] : v[0], k1 = h1 ? v[3] : v[1];
    k0 += __shfl_xor_sync(0xffffffffu, h1 ? v[0] : v[2], WL / 2);
    k1 += __shfl_xor_sync(0xffffffffu, h1 ? v[1] : v[3], WL / 2);
    const bool h2 = lane & (WL / 4);
    y = (h2 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, h2 ? k0 : k1, WL / 4);
#pragma unroll
    for (int off = WL / 8; off > 0; off >>= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
  } else {
    const bool h1 = lane & (WL / 2);
    y = (h1 ? v[1] : v[0]) + __shfl_xor_sync(0xffffffffu, h1 ? v[0] : v[1], WL / 2);
#pragma unroll
    for (int off = WL / 4; off > 0; off >>= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
  }
  return y;
}
struct SumOp { __device__ float operator()(float a, float b) const { return a + b; } };

// GQ contiguous state-vector values of run `base` (swizzled shared memory).
template <class C>
__device__ __forceinline__ void read_run(const float *vec, int base, float *dst) {
  constexpr int GQ = C::GQ;
  if constexpr (GQ == 1) {
    dst[0] = vec[swz<C::SWZ>(base)];
  } else if constexpr (GQ == 2) {
    const float2 v = *reinterpret_cast<const float2 *>(vec + swz<C::SWZ>(base));
    dst[0] = v.x; dst[1] = v.y;
  } else {
#pragma unroll
    for (int q = 0; q < GQ / 4; ++q) {
      const float4 v = *reinterpret_cast<const float4 *>(vec + swz<C::SWZ>(base + 4 * q));
      dst[4 * q] = v.x; dst[4 * q + 1] = v.y; dst[4 * q + 2] = v.z; dst[4 * q + 3] = v.w;
    }
  }
}

template <class C>
__device__ __forceinline__ void write_run(float *vec, int base, const float *src) {
  constexpr int GQ = C::GQ;
  if constexpr (GQ == 1) {
    vec[swz<C::SWZ>(base)] = src[0];
  } else if constexpr (GQ == 2) {
    *reinterpret_cast<float2 *>(vec + swz<C::SWZ>(base)) = make_float2(src[0], src[1]);
  } else {
#pragma unroll
    for (int q = 0; q < GQ / 4; ++q)
      *reinterpret_cast<float4 *>(vec + swz<C::SWZ>(base + 4 * q)) =
          make_float4(src[4 * q], src[4 * q + 1], src[4 * q + 2], src[4 * q + 3]);
  }
}

// N (1, 2 or 4) contiguous state-vector values at base (N | base).
template <class C, int N>
__device__ __forceinline__ void write_sub(float *vec, int base, const float *src) {
  if constexpr (N == 1) {
    vec[swz<C::SWZ>(base)] = src[0];
  } else if constexpr (N == 2) {
    *reinterpret_cast<float2 *>(vec + swz<C::SWZ>(base)) = make_float2(src[0], src[1]);
  } else {
    *reinterpret_cast<float4 *>(vec + swz<C::SWZ>(base)) = make_float4(src[0], src[1], src[2], src[3]);
  }
}

template <class C>
__global__ void __launch_bounds__(C::NT, C::MINB)
bcjr_kernel(const float *__restrict__ s, const float *__restrict__ Dw, int64_t n_seq, int T,
            float kappa, float two_over_temp, float cmin, float cmax_code,
            const float *__restrict__ vgrad, const float *__restrict__ soft_in,
            float *__restrict__ soft_out, float *__restrict__ logz_out,
            float *__restrict__ grad_out, float *__restrict__ ws) {
  constexpr int NG = C::NG, G = C::G, GQ = C::GQ, TPS = C::TPS, NB = C::NBUF, NV = C::NV;
  constexpr int NPART = C::NPART, SPC = C::SPC, PREC = C::PREC, NCH = C::SPILL / 4;
  constexpr bool GRAD = C::GRAD;
  extern __shared__ __align__(16) float smem[];
  float *Vall = smem;                                      // [SPC][NB][NV][NG]
  float2 *Csm = reinterpret_cast<float2 *>(Vall + SPC * C::VPS * NG);  // [HS][G][TPS]
  float *ssm = reinterpret_cast<float *>(Csm + (C::TMEMC ? 0 : C::HS * G * TPS));  // [SPC][256]
  float *ksm = ssm + SPC * 256;                            // [SPC][256] kappa * D_t
  float *vsm = ksm + SPC * 256;                            // GRAD: v, soft rows
  float *fsm = vsm + (GRAD ? SPC * 256 : 0);
  float *cah = fsm + (GRAD ? SPC * 256 : 0);               // [SPC][256] CA_t - CA_{t-1}
  float *part = cah + SPC * 256;                           // [2][SPC][NPART][PREC]

  const int tid = threadIdx.x;
  const int ls = tid / TPS, w = tid - ls * TPS;
  const int lane = tid & 31;
  const int pidx = TPS >= 32 ? (w >> 5) : 0;
  const bool plead = TPS >= 32 ? (lane == 0) : (w == 0);

  CodeRegs<C> cv;
#pragma unroll
  for (int h = 0; h < C::HREG; ++h)
#pragma unroll
    for (int i = 0; i < G; ++i)
      cv[h][i] = f2(one_mad_f32((uint32_t)(2 * h * NG + G * w + i)),
                    one_mad_f32((uint32_t)((2 * h + 1) * NG + G * w + i)));
  __shared__ uint32_t tmem_base;
  uint32_t taddr = 0;
  if constexpr (C::TMEMC) {
    // one allocation per CTA; thread (warp, lane) owns TMEM lane 32 (warp % 4) +
    // lane, columns (warp / 4) TCPT .. + TCPT - 1
    if (tid < 32) tmem_alloc(&tmem_base, C::TCOLS);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const int warp = tid >> 5;
    taddr = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)((warp >> 2) * C::TCPT);
    for (int h = C::HREG; h < 2; ++h)
      for (int i = 0; i < G; i += 4) {
        float v[8];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          v[2 * n] = one_mad_f32((uint32_t)(2 * h * NG + G * w + i + n));
          v[2 * n + 1] = one_mad_f32((uint32_t)((2 * h + 1) * NG + G * w + i + n));
        }
        tmem_st8(taddr + 2 * ((h - C::HREG) * G + i), v);
      }
    tmem_wait_st();
  } else if (ls == 0) {
    for (int h = C::HREG; h < 2; ++h)
      for (int i = 0; i < G; ++i)
        Csm[((h - C::HREG) * G + i) * TPS + w] =
            make_float2(one_mad_f32((uint32_t)(2 * h * NG + G * w + i)),
                        one_mad_f32((uint32_t)((2 * h + 1) * NG + G * w + i)));
  }
  const CodeSrc<C> codes{cv, Csm, taddr, w};

  // thread-private spill: [T][NCH][TPS] float4; step t holds A_t (and Phi_t)
  // at this thread's groups r = a*NG/4 + GQ*w + k, flattened as a*GQ + k.
  float4 *spill = reinterpret_cast<float4 *>(ws + (size_t)(blockIdx.x * SPC + ls) *
                                                      C::ws_floats_per_slot(T));
  // then [T][NPART] records of NQS sums (numerator, denominator; gradient:
  // the two moments), read back once the backward is done
  float *sums = reinterpret_cast<float *>(spill) + (size_t)T * NV * NG;
  auto prec = [&](int parity) { return part + ((parity * SPC + ls) * NPART) * PREC; };

  if constexpr (C::NAMED || C::WARPSEQ) __syncthreads();   // the shared code values are in place
  // targets (and curvature, cotangent, centre) of step t of sequence row l
  auto load_row = [&](int l, int t, int64_t base) {
    const int64_t sq = base + l;
    const bool ok = sq < n_seq;
    ssm[l * 256 + t] = ok ? s[sq * T + t] : 0.0f;
    ksm[l * 256 + t] = kappa * ((ok && Dw) ? Dw[sq * T + t] : 1.0f);
    if (GRAD) {
      vsm[l * 256 + t] = ok ? vgrad[sq * T + t] : 0.0f;
      // centre of the covariance (any per-step constant is exact): the
      // forward soft codeword when given, else the target clamped to the
      // code range, which keeps F small for targets far outside it
      fsm[l * 256 + t] = ok ? (soft_in ? soft_in[sq * T + t]
                                       : fminf(fmaxf(s[sq * T + t], cmin), cmax_code))
                            : 0.0f;
    }
  };
  for (int64_t base = (int64_t)blockIdx.x * SPC; base < n_seq; base += (int64_t)gridDim.x * SPC) {
    const int64_t seq = base + ls;
    const bool active = seq < n_seq;
    seq_sync<C>(ls);                                       // previous sequence fully done
    if constexpr (C::NAMED || C::WARPSEQ) {                // each sequence loads its own rows
      for (int t = w; t < T; t += TPS) load_row(ls, t, base);
    } else {
      for (int x = tid; x < SPC * T; x += C::NT) load_row(x / T, x % T, base);
    }
    float *V = Vall + ls * C::VPS * NG;
    // the message (A or B) and expectation (Phi or Psi) vectors of step x >= -1
    auto msg_buf = [&](int x) -> float * {
      return C::MSG2 ? V + (x & 1) * NG : V + ((x + NB) % NB) * NV * NG;
    };
    auto exp_buf = [&](int x) -> float * {
      return C::MSG2 ? V + 2 * NG : V + ((x + NB) % NB) * NV * NG + NG;
    };
    if constexpr (C::MSG2) {
      for (int x = w; x < NG; x += TPS) {                 // A_0 = 0, Phi_0 = 0
        msg_buf(0)[x] = 0.0f;
        exp_buf(0)[x] = 0.0f;
      }
    } else {
      for (int x = w; x < NV * NG; x += TPS) V[x] = 0.0f;   // A_0 = 0 (and Phi_0 = 0)
    }
    if constexpr (C::NAMED || C::WARPSEQ) {
      for (int x = w; x < NPART * PREC; x += TPS) { prec(0)[x] = 0.0f; prec(1)[x] = 0.0f; }
    } else {
      for (int x = tid; x < 2 * SPC * NPART * PREC; x += C::NT) part[x] = 0.0f;
    }
    seq_sync<C>(ls);

    // ---------------- forward ----------------
    // A_t is stored relative to CA_t = c_0 + ... + c_{t-1}, c_t = max of stored A_t.
    // CA itself is needed only for log Z; the combine takes the increments
    // c_{t-1} = CA_t - CA_{t-1} (cah[t]), because CA can be huge (it grows by
    // up to kappa max(e) per step) while what the combine needs is small.
    float CA = 0.0f, cmax = 0.0f;
    if (w == 0) cah[ls * 256] = 0.0f;
    // lazyA (the L = 16 kernels): the loop stops before step T, whose spill of
    // A_{T-1} (and Phi_{T-1}) follows the loop; inside it A_{t-1} is read (and
    // spilled) block by block in the step itself, so that its 4G values are
    // not all held in registers at once (L = 16 soft pass: 64.4 -> 59.8 ms on
    // 4,440 sequences)
    constexpr bool lazyA = C::MSG2 || (!GRAD && C::TMEMC && NB == 2 && GQ % 4 == 0);
    for (int t = 1; t <= (lazyA ? T - 1 : T); ++t) {
      const float *Ai = C::MSG2 ? msg_buf(t - 1) : V + ((t - 1) % NB) * NV * NG;
      const float *Fi = C::MSG2 ? exp_buf(t - 1) : Ai + NG;
      float ain[4][GQ], fin[GRAD ? 4 : 1][GQ];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        if (!lazyA) read_run<C>(Ai, a * (NG / 4) + GQ * w, ain[a]);
        if (GRAD) read_run<C>(Fi, a * (NG / 4) + GQ * w, fin[a < (GRAD ? 4 : 1) ? a : 0]);
      }
      cmax = 0.0f;
      if (t > 1) {
        const float *pp = prec((t - 1) & 1);
        cmax = pp[0];
#pragma unroll
        for (int x = 1; x < NPART; ++x) cmax = fmaxf(cmax, pp[x * PREC]);
      }
      {   // spill A_{t-1} (and Phi_{t-1}) at this thread's groups
        float flat[C::SPILL];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int k = 0; k < GQ; ++k) {
            flat[a * GQ + k] = lazyA ? 0.0f : ain[a][k];
            if (GRAD) flat[G + a * GQ + k] = fin[a < (GRAD ? 4 : 1) ? a : 0][k];
          }
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          if (!lazyA || 4 * c >= G)
            spill[((size_t)(t - 1) * NCH + c) * TPS + w] =
                make_float4(flat[4 * c], flat[4 * c + 1], flat[4 * c + 2], flat[4 * c + 3]);
      }
      if (t == T) break;
      if (w == 0) cah[ls * 256 + t] = cmax;
      if (NB == 1) seq_sync<C>(ls);
      CA += cmax;
      float *Ao = C::MSG2 ? msg_buf(t) : V + (t % NB) * NV * NG;
      float *Fo = C::MSG2 ? exp_buf(t) : Ao + NG;
      const float sv = ssm[ls * 256 + t - 1];
      const float vv = GRAD ? vsm[ls * 256 + t - 1] : 0.0f;
      const float fv = GRAD ? fsm[ls * 256 + t - 1] : 0.0f;
      float tmax = -INFINITY;
      // emissions relative to r, the target clamped to the code range:
      // -kappa (c - s)^2 = d (-kappa d + beta) - kappa (r - s)^2 with d = c - r,
      // beta = 2 kappa (s - r).  The last term is the same for every state of
      // the step (posteriors unchanged; log Z gets it back), and for a target
      // inside the range r = s, beta = +0 and the two FMAs round exactly like
      // the plain -kappa d d.  Outside it the states that compete carry small,
      // accurately rounded emissions.
      const float rv = fminf(fmaxf(sv, cmin), cmax_code);
      const f2_t sv2 = f2(rv, rv), cm2 = f2(cmax, cmax);
      const f2_t nk2 = f2(-ksm[ls * 256 + t - 1], -ksm[ls * 256 + t - 1]);
      const float beta = 2.0f * ksm[ls * 256 + t - 1] * (sv - rv);
      const f2_t b2 = f2(beta, beta);
      if constexpr (!GRAD) {
        // code pairs of group block q + 1 are loaded from tensor memory while
        // block q computes; the wait at the end of block q completes them
        // (L = 16 soft pass 59.8 -> 59.2 ms on 4,440 sequences; the same in
        // the backward, one 32-column block ahead, measured slower)
        float rc[2][2][8];
        if constexpr (C::TMEMC && C::HREG == 0) {
          tmem_ld8(taddr + 0, rc[0][0]);
          tmem_ld8(taddr + 2 * G, rc[0][1]);
          tmem_wait_ld();
        }
#pragma unroll
        for (int q = 0; q < GQ; ++q) {
          if (lazyA && (q & 3) == 0) {                      // A_{t-1} for groups 4q .. 4q + 15
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const float4 v =
                  *reinterpret_cast<const float4 *>(Ai + swz<C::SWZ>(a * (NG / 4) + GQ * w + q));
              ain[a][q] = v.x; ain[a][(q + 1) % GQ] = v.y;
              ain[a][(q + 2) % GQ] = v.z; ain[a][(q + 3) % GQ] = v.w;
              spill[((size_t)(t - 1) * NCH + (a * GQ + q) / 4) * TPS + w] = v;
            }
          }
          // inputs of group 4q + r from predecessor digits (0, 1) and (2, 3)
          const f2_t am0 = f2sub(f2(ain[0][q], ain[1][q]), cm2);
          const f2_t am1 = f2sub(f2(ain[2][q], ain[3][q]), cm2);
          float outA[4];
          f2_t cq0[4], cq1[4];
          if constexpr (C::TMEMC && C::HREG == 0) {
            if (q + 1 < GQ) {
              tmem_ld8(taddr + 2 * (4 * (q + 1)), rc[(q + 1) & 1][0]);
              tmem_ld8(taddr + 2 * (G + 4 * (q + 1)), rc[(q + 1) & 1][1]);
            }
#pragma unroll
            for (int n = 0; n < 4; ++n) {
              cq0[n] = f2(rc[q & 1][0][2 * n], rc[q & 1][0][2 * n + 1]);
              cq1[n] = f2(rc[q & 1][1][2 * n], rc[q & 1][1][2 * n + 1]);
            }
          } else {
            codes.both_pairs4(4 * q, cq0, cq1);
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const f2_t d0 = f2sub(cq0[r], sv2);
            const f2_t d1 = f2sub(cq1[r], sv2);
            const f2_t x0 = f2fma(d0, f2fma(nk2, d0, b2), am0);
            const f2_t x1 = f2fma(d1, f2fma(nk2, d1, b2), am1);
            outA[r] = lse4_base2(f2lo(x0), f2hi(x0), f2lo(x1), f2hi(x1));
            tmax = fmaxf(tmax, outA[r]);
          }
          *reinterpret_cast<float4 *>(Ao + swz<C::SWZ>(G * w + 4 * q)) =
              make_float4(outA[0], outA[1], outA[2], outA[3]);
          if constexpr (C::TMEMC && C::HREG == 0) tmem_wait_ld();
        }
      } else {
        const f2_t vv2 = f2(vv, vv), vf2 = f2(vv * fv, vv * fv);
#pragma unroll
        for (int q = 0; q < GQ; ++q) {
          if (lazyA && (q & 3) == 0) {                      // A_{t-1} for groups 4q .. 4q + 15
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const float4 v =
                  *reinterpret_cast<const float4 *>(Ai + swz<C::SWZ>(a * (NG / 4) + GQ * w + q));
              ain[a][q] = v.x; ain[a][(q + 1) % GQ] = v.y;
              ain[a][(q + 2) % GQ] = v.z; ain[a][(q + 3) % GQ] = v.w;
              spill[((size_t)(t - 1) * NCH + (a * GQ + q) / 4) * TPS + w] = v;
            }
          }
          const f2_t am0 = f2sub(f2(ain[0][q], ain[1][q]), cm2);
          const f2_t am1 = f2sub(f2(ain[2][q], ain[3][q]), cm2);
          const f2_t ph0 = f2sub(f2(fin[0][q], fin[1][q]), vf2);
          const f2_t ph1 = f2sub(f2(fin[2][q], fin[3][q]), vf2);
          float outA[4], outF[4];
          f2_t cq0[4], cq1[4];
          codes.both_pairs4(4 * q, cq0, cq1);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const f2_t c0 = cq0[r];
            const f2_t c1 = cq1[r];
            const f2_t d0 = f2sub(c0, sv2), d1 = f2sub(c1, sv2);
            const f2_t x0 = f2fma(d0, f2fma(nk2, d0, b2), am0);
            const f2_t x1 = f2fma(d1, f2fma(nk2, d1, b2), am1);
            const f2_t z0 = f2fma(vv2, c0, ph0);            // phi_{t-1}(p) = Phi + v (c - soft)
            const f2_t z1 = f2fma(vv2, c1, ph1);
            const float mx = fmaxf(fmaxf(f2lo(x0), f2hi(x0)), fmaxf(f2lo(x1), f2hi(x1)));
            const f2_t mx2 = f2(mx, mx);
            const f2_t e0 = f2sub(x0, mx2), e1 = f2sub(x1, mx2);
            const f2_t u0 = f2(ex2(f2lo(e0)), ex2(f2hi(e0)));
            const f2_t u1 = f2(ex2(f2lo(e1)), ex2(f2hi(e1)));
            const f2_t su = f2add(u0, u1);
            const f2_t sz = f2fma(u1, z1, f2mul(u0, z0));
            const float S = f2lo(su) + f2hi(su);
            outA[r] = mx + lg2(S);
            tmax = fmaxf(tmax, outA[r]);
            outF[r] = (f2lo(sz) + f2hi(sz)) * rcp(S);
          }
          *reinterpret_cast<float4 *>(Ao + swz<C::SWZ>(G * w + 4 * q)) =
              make_float4(outA[0], outA[1], outA[2], outA[3]);
          *reinterpret_cast<float4 *>(Fo + swz<C::SWZ>(G * w + 4 * q)) =
              make_float4(outF[0], outF[1], outF[2], outF[3]);
        }
      }
      tmax = seq_max<TPS>(tmax);
      if (plead) prec(t & 1)[pidx * PREC] = tmax;
      seq_sync<C>(ls);
    }
    if constexpr (lazyA) {                                   // step T: spill A_{T-1}, Phi_{T-1}
      cmax = 0.0f;
      if (T > 1) {
        const float *pp = prec((T - 1) & 1);
        cmax = pp[0];
#pragma unroll
        for (int x = 1; x < NPART; ++x) cmax = fmaxf(cmax, pp[x * PREC]);
      }
      const float *Ai = msg_buf(T - 1);
      const float *Fi = exp_buf(T - 1);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < GQ; q += 4) {
          const float4 va = *reinterpret_cast<const float4 *>(Ai + swz<C::SWZ>(a * (NG / 4) + GQ * w + q));
          spill[((size_t)(T - 1) * NCH + (a * GQ + q) / 4) * TPS + w] = va;
          if constexpr (GRAD) {
            const float4 vf = *reinterpret_cast<const float4 *>(Fi + swz<C::SWZ>(a * (NG / 4) + GQ * w + q));
            spill[((size_t)(T - 1) * NCH + (G + a * GQ + q) / 4) * TPS + w] = vf;
          }
        }
    }
    // CA = CA_{T-1}; cmax = max of stored A_{T-1}; spill step T-1 holds A_{T-1}.

    // ---------------- log2 Z = LSE over all states at T-1 ----------------
    float log2Z, log2Zrel;
    {
      const float sT = ssm[ls * 256 + T - 1];
      const float rT = fminf(fmaxf(sT, cmin), cmax_code);          // as in the forward
      const float bT = 2.0f * ksm[ls * 256 + T - 1] * (sT - rT);
      float vals[4][GQ], vmax = -INFINITY;
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        float av[GQ];
#pragma unroll
        for (int q = 0; q < (GQ + 3) / 4; ++q) {
          const int f = a * GQ + 4 * q;
          const float4 v = spill[((size_t)(T - 1) * NCH + (f >> 2)) * TPS + w];
          const float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 4 && 4 * q + k < GQ; ++k) av[4 * q + k] = e4[(f & 3) + k];
        }
#pragma unroll
        for (int k = 0; k < GQ; ++k) {
          float y[4];
          f2_t cp[4];
          codes.template pairs<4>(a >> 1, 4 * k, cp);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float d = ((a & 1) ? f2hi(cp[b]) : f2lo(cp[b])) - rT;
            y[b] = fmaf(-ksm[ls * 256 + T - 1], d, bT) * d;
          }
          const float mx = fmaxf(fmaxf(y[0], y[1]), fmaxf(y[2], y[3]));
          const float S = ex2(y[0] - mx) + ex2(y[1] - mx) + ex2(y[2] - mx) + ex2(y[3] - mx);
          vals[a][k] = (av[k] - cmax) + mx + lg2(S);
          vmax = fmaxf(vmax, vals[a][k]);
        }
      }
      vmax = lane_reduce<TPS>(vmax, MaxOp());
      float *pp = prec(0);
      if (plead) pp[pidx * PREC + 5] = vmax;
      seq_sync<C>(ls);
      vmax = pp[5];
#pragma unroll
      for (int x = 1; x < NPART; ++x) vmax = fmaxf(vmax, pp[x * PREC + 5]);
      float sum = 0.0f;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int k = 0; k < GQ; ++k) sum += ex2(vals[a][k] - vmax);
      sum = lane_reduce<TPS>(sum, SumOp());
      if (plead) pp[pidx * PREC + 6] = sum;
      seq_sync<C>(ls);
      float tot = 0.0f;
#pragma unroll
      for (int x = 0; x < NPART; ++x) tot += pp[x * PREC + 6];
      log2Zrel = vmax + lg2(tot) + cmax;                  // log2 Z - CA_{T-1}
      log2Z = log2Zrel + CA;
    }
    if (w == 0 && active && logz_out) {
      // add back kappa D_u (r_u - s_u)^2, removed from every walk's log2
      // weight at the steps whose target lies outside the code range
      double removed = 0.0;
      for (int u = 0; u < T; ++u) {
        const float su = ssm[ls * 256 + u];
        const double e = (double)fminf(fmaxf(su, cmin), cmax_code) - (double)su;
        removed += (double)ksm[ls * 256 + u] * e * e;
      }
      logz_out[seq] = (float)(((double)log2Z - removed) * 0.69314718055994531);
    }

    // ---------------- backward + combine ----------------
    // B_t is stored relative to DB_t (sum of the maxima removed); the combine
    // at step tc uses K = log2Z - CA_tc - DB_tc so that the group weights are
    // the posteriors themselves (sum ~ 1).  K is carried as a running value,
    // K_{tc-1} = K_tc + (CA_tc - CA_{tc-1}) - (DB_{tc-1} - DB_tc), starting
    // from log2 Z - CA_{T-1}, so no two huge sums are ever subtracted.
    float *Bv = V;
    if constexpr (C::MSG2) {
      for (int x = w; x < NG; x += TPS) {                 // B_{T-1} = 0, Psi_{T-1} = 0
        msg_buf(T - 1)[x] = 0.0f;
        exp_buf(T - 1)[x] = 0.0f;
      }
    } else {
      for (int x = w; x < NV * NG; x += TPS) Bv[((T - 1) % NB) * NV * NG + x] = 0.0f;
    }
    seq_sync<C>(ls);
    float Krun = log2Zrel;
    // soft pass with G <= 16: the thread's spilled A of each backward step
    // sits in registers, loaded one step ahead
    constexpr bool PREFETCH = !GRAD && G <= 16;
    [[maybe_unused]] float4 avn[PREFETCH ? NCH : 1];
    if constexpr (PREFETCH) {
#pragma unroll
      for (int c = 0; c < NCH; ++c) avn[c] = spill[((size_t)(T - 1) * NCH + c) * TPS + w];
    }
    for (int t = T - 2; t >= -1; --t) {
      const int tc = t + 1;                                  // combine step
      // this thread's spilled A_tc values (issued first: they come from HBM)
      // (the gradient pass carries twice the values and would spill registers)
      float4 avq[PREFETCH ? NCH : 1];
      if constexpr (PREFETCH) {                              // this step's, loaded a step ago
#pragma unroll
        for (int c = 0; c < NCH; ++c) avq[c] = avn[c];
        if (tc > 0) {
#pragma unroll
          for (int c = 0; c < NCH; ++c) avn[c] = spill[((size_t)(tc - 1) * NCH + c) * TPS + w];
        }
      }
      // the next step's spilled chunks are read a whole step from now: start
      // bringing them on chip (register prefetch covers the small soft case)
      if constexpr (!PREFETCH) {
        if (tc > 0) {
#pragma unroll
          for (int c = 0; c < NCH; ++c)
            prefetch_global<TCQ_SPILL_PREFETCH_LEVEL>(&spill[((size_t)(tc - 1) * NCH + c) * TPS + w]);
        }
      }
      const float *Bi = C::MSG2 ? msg_buf(tc) : Bv + (tc % NB) * NV * NG;
      const float *Pi = C::MSG2 ? exp_buf(tc) : Bi + NG;
      float bin[C::MSG2 ? 1 : G], pin[GRAD ? G : 1];
#pragma unroll
      for (int q = 0; q < GQ; ++q) {
        if constexpr (!C::MSG2) {                            // MSG2: read where used
          const float4 v = *reinterpret_cast<const float4 *>(Bi + swz<C::SWZ>(G * w + 4 * q));
          bin[4 * q] = v.x; bin[4 * q + 1] = v.y; bin[4 * q + 2] = v.z; bin[4 * q + 3] = v.w;
        }
        if (GRAD) {
          const float4 f = *reinterpret_cast<const float4 *>(Pi + swz<C::SWZ>(G * w + 4 * q));
          pin[4 * q] = f.x; pin[4 * q + 1] = f.y; pin[4 * q + 2] = f.z; pin[4 * q + 3] = f.w;
        }
      }
      float dprev = 0.0f;                                    // max of stored B_tc
      if (tc < T - 1) {
        const float *pp = prec((tc + 1) & 1);
        dprev = pp[0];
#pragma unroll
        for (int x = 1; x < NPART; ++x) dprev = fmaxf(dprev, pp[x * PREC]);
      }
      if (NB == 1) seq_sync<C>(ls);
      const float K = Krun;
      Krun += cah[ls * 256 + tc] - dprev;
      const float s_tc = ssm[ls * 256 + tc];
      const float sv = fminf(fmaxf(s_tc, cmin), cmax_code);          // r, as in the forward
      const float vv = GRAD ? vsm[ls * 256 + tc] : 0.0f;
      const float fv = GRAD ? fsm[ls * 256 + tc] : 0.0f;
      float *Bo = C::MSG2 ? msg_buf(t) : Bv + ((t + NB) % NB) * NV * NG;
      float *Po = C::MSG2 ? exp_buf(t) : Bo + NG;
      float num = 0.0f, den = 0.0f, n1 = 0.0f, n2 = 0.0f, tmax = -INFINITY;
      const f2_t sv2 = f2(sv, sv), nk2 = f2(-ksm[ls * 256 + tc], -ksm[ls * 256 + tc]);
      const float beta = 2.0f * ksm[ls * 256 + tc] * (s_tc - sv);
      const f2_t b2 = f2(beta, beta);
      const f2_t K2 = f2(K, K), dp2 = f2(dprev, dprev), vv2 = f2(vv, vv);
      f2_t num2 = f2(0.0f, 0.0f), den2 = num2, n12 = num2, n22 = num2;
      // KB values of this thread's spilled vector at flat index f (KB | f)
      // sub-run width 2.  Measured at L = 16: in the gradient pass, which
      // holds Psi of 32 groups across the step's first barrier, 1 spilled
      // fewer registers but read every spilled float4 twice (24.2 vs 23.5 ms
      // on 1,036 sequences); in the soft pass, 4 ran 60.0 against 58.2 ms on
      // 4,440 sequences
      constexpr int KB = GQ < 2 ? GQ : 2;
      auto spilled_run = [&](int f, float *dst) {
        float4 v;
        if constexpr (PREFETCH) v = avq[PREFETCH ? (f >> 2) : 0];
        else v = spill[((size_t)tc * NCH + (f >> 2)) * TPS + w];
        const float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < KB; ++j) dst[j] = e4[(f & 3) + j];
      };
      const float nvf = -vv * fv;
      // digit pair h: groups r = a NG/4 + GQ w + k of digits a = 2h, 2h+1 side by
      // side; their successors 4r + b share the B_{tc+1} value bin[4k + b]
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int kb = 0; kb < GQ / KB; ++kb) {
          float avl[KB], avh[KB], fal[GRAD ? KB : 1], fah[GRAD ? KB : 1];
          spilled_run(2 * h * GQ + KB * kb, avl);
          spilled_run((2 * h + 1) * GQ + KB * kb, avh);
          if constexpr (GRAD) {
            spilled_run(G + 2 * h * GQ + KB * kb, fal);
            spilled_run(G + (2 * h + 1) * GQ + KB * kb, fah);
          }
          float outL[KB], outH[KB], outPL[GRAD ? KB : 1], outPH[GRAD ? KB : 1];
          // code pairs (h, 4k + b) of this block: one tensor-memory load for the
          // block, else four pairs per group index as it is reached
          constexpr bool BLK = C::TMEMC && KB >= 2;
          f2_t cb[BLK ? 4 * KB : 1];
          if constexpr (BLK) codes.template pairs<BLK ? 4 * KB : 4>(h, 4 * KB * kb, cb);
#pragma unroll
          for (int j = 0; j < KB; ++j) {
            const int k = KB * kb + j;
            f2_t cc[4], y[4];
            if constexpr (BLK) {
#pragma unroll
              for (int b = 0; b < 4; ++b) cc[b] = cb[BLK ? 4 * j + b : 0];
            } else {
              codes.template pairs<4>(h, 4 * k, cc);
            }
            float bk[4];                                     // B_{tc+1} of the successors
            if constexpr (C::MSG2) {
              const float4 v = *reinterpret_cast<const float4 *>(Bi + swz<C::SWZ>(G * w + 4 * k));
              bk[0] = v.x; bk[1] = v.y; bk[2] = v.z; bk[3] = v.w;
            } else {
#pragma unroll
              for (int b = 0; b < 4; ++b) bk[b] = bin[C::MSG2 ? 0 : 4 * k + b];
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const f2_t d = f2sub(cc[b], sv2);
              y[b] = f2fma(d, f2fma(nk2, d, b2), f2(bk[b], bk[b]));
            }
            if constexpr (C::POSTB) {
              // exponents taken against the combine's reference K: with
              // aK = A_tc(r) - K, 2^(aK + y_b) is the posterior of successor
              // state 4r + b at step tc (at most 1, so no maximum is needed).
              // Their sums give the combine's weights directly,
              // B_t(r) = lg2(sum) - aK - dp and (gradient) Psi_t(r) = the
              // weighted mean of z: four ex2 and one lg2 per group, where a
              // maximum-relative log-sum-exp and a separate group weight take
              // five ex2.  A term that underflows is a state whose posterior is
              // below 2^-126; the paths through it change no output.
              const f2_t aK = f2sub(f2(avl[j], avh[j]), K2);
              f2_t S, sc, sz, scz;
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const f2_t e = f2add(y[b], aK);
                const f2_t v = f2(ex2(f2lo(e)), ex2(f2hi(e)));
                S = b == 0 ? v : f2add(S, v);
                if constexpr (!GRAD) {
                  sc = b == 0 ? f2mul(v, cc[b]) : f2fma(v, cc[b], sc);
                } else {
                  const f2_t vc = f2mul(v, cc[b]);
                  sc = b == 0 ? vc : f2add(sc, vc);
                  // z_b = psi_{tc}(succ) + v_tc (c_b - soft_tc)
                  const float pz = pin[4 * k + b] + nvf;
                  const f2_t z = f2fma(vv2, cc[b], f2(pz, pz));
                  sz = b == 0 ? f2mul(v, z) : f2fma(v, z, sz);
                  scz = b == 0 ? f2mul(vc, z) : f2fma(vc, z, scz);
                }
              }
              const f2_t ob = f2sub(f2(lg2(f2lo(S)), lg2(f2hi(S))), f2add(aK, dp2));
              outL[j] = f2lo(ob);
              outH[j] = f2hi(ob);
              tmax = fmaxf(tmax, fmaxf(outL[j], outH[j]));
              den2 = f2add(den2, S);
              num2 = f2add(num2, sc);
              if constexpr (GRAD) {
                // Psi_t(r) = sz / S, and 0 where every successor underflowed
                // (their weight is 0 wherever the value is used)
                outPL[j] = f2lo(S) > 0.0f ? f2lo(sz) * rcp(f2lo(S)) : 0.0f;
                outPH[j] = f2hi(S) > 0.0f ? f2hi(sz) * rcp(f2hi(S)) : 0.0f;
                const f2_t fa2 = f2(fal[j], fah[j]);
                n12 = f2add(n12, f2fma(fa2, S, sz));
                n22 = f2add(n22, f2fma(fa2, sc, scz));
              }
            } else {
              // maximum-relative log-sum-exp and a separate group weight: the
              // B recursion does not wait on the spilled A (L = 8, where one
              // warp per scheduler leaves that latency exposed)
              const float mxl = fmaxf(fmaxf(f2lo(y[0]), f2lo(y[1])), fmaxf(f2lo(y[2]), f2lo(y[3])));
              const float mxh = fmaxf(fmaxf(f2hi(y[0]), f2hi(y[1])), fmaxf(f2hi(y[2]), f2hi(y[3])));
              const f2_t mx2 = f2(mxl, mxh);
              // sums over the four successors, accumulated one successor at a
              // time (fewer live registers than four separate weights)
              f2_t su, sc, sz, scz;
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const f2_t e = f2sub(y[b], mx2);
                const f2_t u = f2(ex2(f2lo(e)), ex2(f2hi(e)));
                su = b == 0 ? u : f2add(su, u);
                if constexpr (!GRAD) {
                  sc = b == 0 ? f2mul(u, cc[b]) : f2fma(u, cc[b], sc);
                } else {
                  const f2_t uc = f2mul(u, cc[b]);
                  sc = b == 0 ? uc : f2add(sc, uc);
                  // z_b = psi_{tc}(succ) + v_tc (c_b - soft_tc)
                  const float pz = pin[4 * k + b] + nvf;
                  const f2_t z = f2fma(vv2, cc[b], f2(pz, pz));
                  sz = b == 0 ? f2mul(u, z) : f2fma(u, z, sz);
                  scz = b == 0 ? f2mul(uc, z) : f2fma(uc, z, scz);
                }
              }
              const f2_t ob = f2add(f2sub(mx2, dp2), f2(lg2(f2lo(su)), lg2(f2hi(su))));
              outL[j] = f2lo(ob);
              outH[j] = f2hi(ob);
              tmax = fmaxf(tmax, fmaxf(outL[j], outH[j]));
              const f2_t wv = f2add(f2sub(f2(avl[j], avh[j]), K2), mx2);
              const f2_t wgt = f2(ex2(f2lo(wv)), ex2(f2hi(wv)));
              den2 = f2fma(wgt, su, den2);
              num2 = f2fma(wgt, sc, num2);
              if constexpr (GRAD) {
                const f2_t op = f2mul(sz, f2(rcp(f2lo(su)), rcp(f2hi(su))));
                outPL[j] = f2lo(op);
                outPH[j] = f2hi(op);
                const f2_t fa2 = f2(fal[j], fah[j]);
                n12 = f2fma(wgt, f2fma(fa2, su, sz), n12);
                n22 = f2fma(wgt, f2fma(fa2, sc, scz), n22);
              }
            }
          }
          if (t >= 0) {
            const int bl = 2 * h * (NG / 4) + GQ * w + KB * kb, bh = bl + NG / 4;
            write_sub<C, KB>(Bo, bl, outL);
            write_sub<C, KB>(Bo, bh, outH);
            if constexpr (GRAD) {
              write_sub<C, KB>(Po, bl, outPL);
              write_sub<C, KB>(Po, bh, outPH);
            }
          }
        }
      }
      num = f2lo(num2) + f2hi(num2);
      den = f2lo(den2) + f2hi(den2);
      if constexpr (GRAD) {
        n1 = f2lo(n12) + f2hi(n12);
        n2 = f2lo(n22) + f2hi(n22);
      }
      tmax = seq_max<TPS>(tmax);
      {
        constexpr int NQ = GRAD ? 4 : 2, WL = TPS < 32 ? TPS : 32;
        float q4[NQ];
        q4[0] = num; q4[1] = den;
        if constexpr (GRAD) { q4[NQ > 2 ? 2 : 0] = n1; q4[NQ > 3 ? 3 : 0] = n2; }
        const float mine = seq_sums<TPS, NQ>(q4, lane);
        const int o = lane & (WL - 1);
        float *pp = prec(tc & 1) + pidx * PREC;
        if ((o & (WL / NQ - 1)) == 0)                                    // num, den (n1, n2)
          sums[((size_t)tc * NPART + pidx) * C::NQS + o / (WL / NQ)] = mine;
        if (plead) pp[0] = tmax;
      }
      seq_sync<C>(ls);
    }
    if (active) {
      // every step's sums are in the workspace (the barrier that closed the
      // last step orders them): the sequence's threads finish them in parallel
      for (int u = w; u < T; u += TPS) {
        float num = 0.0f, den = 0.0f, n1 = 0.0f, n2 = 0.0f;
#pragma unroll
        for (int x = 0; x < NPART; ++x) {
          const float *r = sums + ((size_t)u * NPART + x) * C::NQS;
          num += r[0]; den += r[1];
          if (GRAD) { n1 += r[GRAD ? 2 : 0]; n2 += r[GRAD ? 3 : 0]; }
        }
        if (soft_out) soft_out[seq * T + u] = num / den;
        if (GRAD) {   // 2 D_u / temp = 2 ln2 kappa D_u
          const float inv = 1.0f / den;
          grad_out[seq * T + u] = (1.3862943611198906f * ksm[ls * 256 + u]) *
                                  (n2 * inv - (num * inv) * (n1 * inv));
        }
      }
    }
  }
  if constexpr (C::TMEMC) {                                // every thread is done with its lane
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (tid < 32) tmem_dealloc(tmem_base, C::TCOLS);
  }
}

}  // namespace tcq

using namespace tcq;
using namespace tcq_host;

namespace {

using Soft8 = BcjrCfg<8, 4, 8, 4, 2, false>;
// L = 12: 128 threads / sequence, seven sequences in one 896-thread CTA per SM
// (one wave of 1,036), each stepping on its own named barrier.  Every code
// value is read from one shared-memory copy that the seven share.  Measured
// against seven one-sequence CTAs, each with its own copy (the gradient pass
// then kept digits 0-1 in registers and spilled at 72 registers, and the
// spills missed L1, which the seven copies had taken): soft 0.977 -> 0.883 ms,
// soft + gradient 1.517 -> 1.295 ms on 1,024 sequences.
using Soft12 = BcjrCfg<12, 8, 7, 0, 2, false, 1>;
// L = 16: one 512-thread CTA per SM; all 2^16 code values sit in tensor memory
// (128 columns per thread, the whole 512-column allocation), which leaves the
// shared memory for a double-buffered state vector (one barrier per step).
// Measured against code values half in registers and half in shared memory
// with a single buffer: 32.1 vs 36.2 ms on 2,048 sequences.  At L = 12 (seven
// CTAs per SM) the same layout was 2.2x slower than shared memory, so it is
// used here only.
using Soft16 = BcjrCfg<16, 32, 1, 0, 2, false, 1, true>;
using Grad8 = BcjrCfg<8, 4, 8, 4, 2, true>;
using Grad12 = BcjrCfg<12, 8, 7, 0, 2, true, 1>;
// L = 16 gradient: code values in tensor memory as in the soft pass.  The
// message vector (A forward, B backward) is double-buffered and read block by
// block after the step's first barrier; the expectation vector (Phi, Psi) fits
// only once beside it (192 KiB in all), so it is read ahead of that barrier
// and each step takes two.
using Grad16 = BcjrCfg<16, 32, 1, 0, 1, true, 1, true, true>;

// Smallest and largest fp32 code value of the 2^L states (the same fp64
// division rounded once to fp32 as the kernels' code values), once per L.
void code_bounds(int L, float *lo, float *hi) {
  static float cache[17][2];
  static std::once_flag once[17];
  std::call_once(once[L], [L] {
    float mn = INFINITY, mx = -INFINITY;
    for (uint32_t x = 0; x < (1u << L); ++x) {
      const uint32_t y = x * kLcgMul + kLcgAdd;
      const int bs = (int)(y & 255u) + (int)((y >> 8) & 255u) + (int)((y >> 16) & 255u) + (int)(y >> 24);
      const float v = (float)((double)(bs - 510) / 147.8);
      mn = std::min(mn, v);
      mx = std::max(mx, v);
    }
    cache[L][0] = mn;
    cache[L][1] = mx;
  });
  *lo = cache[L][0];
  *hi = cache[L][1];
}

template <class C>
int grid_for(int64_t n_seq) {
  int dev = 0, per_sm = 0;
  cudaGetDevice(&dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bcjr_kernel<C>, C::NT,
                                                    C::smem_bytes()) != cudaSuccess ||
      per_sm <= 0)
    per_sm = 1;
  const int64_t want = (n_seq + C::SPC - 1) / C::SPC;
  return (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)per_sm * sm_count()));
}

template <class C>
bool set_smem() {
  const size_t smem = C::smem_bytes();
  if (smem <= 48 * 1024) return true;
  return cudaFuncSetAttribute(bcjr_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem) == cudaSuccess;
}

template <class C>
size_t ws_bytes_for(int64_t n_seq, int T) {
  if (!set_smem<C>()) return 0;
  const int grid = grid_for<C>(n_seq);
  return (size_t)grid * C::SPC * C::ws_floats_per_slot(T) * sizeof(float) + 256;
}

template <class C>
tcq_status_t launch(const float *s, const float *D, int64_t n_seq, int T, float kappa,
                    float two_over_temp, const float *v,
                    const float *soft_in, float *soft, float *logz, float *grad, void *ws,
                    size_t ws_bytes, cudaStream_t stream) {
  if (!set_smem<C>()) return TCQ_ERR_CUDA;
  const int grid = grid_for<C>(n_seq);
  const size_t need = (size_t)grid * C::SPC * C::ws_floats_per_slot(T) * sizeof(float);
  if (ws_bytes < need) return TCQ_ERR_WORKSPACE;
  float cmin, cmax;
  code_bounds(C::L, &cmin, &cmax);
  bcjr_kernel<C><<<grid, C::NT, C::smem_bytes(), stream>>>(s, D, n_seq, T, kappa, two_over_temp, cmin, cmax, v,
                                                           soft_in, soft, logz, grad,
                                                           static_cast<float *>(ws));
  return launch_status();
}

}  // namespace

extern "C" size_t tcq_bcjr_workspace_size(const tcq_trellis_t *tr, int64_t n_seq, int with_grad) {
  if (check_trellis(tr) != TCQ_OK || n_seq <= 0) return 256;
  const int T = tr->seq_len;
  if (with_grad) {
    switch (tr->L) {
      case 8: return ws_bytes_for<Grad8>(n_seq, T);
      case 12: return ws_bytes_for<Grad12>(n_seq, T);
      default: return ws_bytes_for<Grad16>(n_seq, T);
    }
  }
  switch (tr->L) {
    case 8: return ws_bytes_for<Soft8>(n_seq, T);
    case 12: return ws_bytes_for<Soft12>(n_seq, T);
    default: return ws_bytes_for<Soft16>(n_seq, T);
  }
}

static bool temp_ok(float temp) { return temp > 0.0f && temp < INFINITY; }

extern "C" tcq_status_t tcq_bcjr_soft(const tcq_trellis_t *tr, const float *s, const float *D,
                                      int64_t n_seq, float temp, float *soft, float *log_z,
                                      void *ws, size_t ws_bytes, void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if (!temp_ok(temp)) return TCQ_ERR_INVALID_ARG;
  if (n_seq < 0 || n_seq > (int64_t)INT32_MAX) return TCQ_ERR_INVALID_ARG;
  if (n_seq == 0) return TCQ_OK;
  if (!s || !soft || !aligned16(s) || !aligned16(soft) || (log_z && !aligned16(log_z)) ||
      (D && !aligned16(D)))
    return TCQ_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TCQ_ERR_WORKSPACE;
  const float kappa = (float)(1.4426950408889634 / (double)temp);
  const float tot = (float)(2.0 / (double)temp);
  cudaStream_t strm = (cudaStream_t)stream;
  const int T = tr->seq_len;
  switch (tr->L) {
    case 8: return launch<Soft8>(s, D, n_seq, T, kappa, tot, nullptr, nullptr, soft, log_z, nullptr, ws, ws_bytes, strm);
    case 12: return launch<Soft12>(s, D, n_seq, T, kappa, tot, nullptr, nullptr, soft, log_z, nullptr, ws, ws_bytes, strm);
    default: return launch<Soft16>(s, D, n_seq, T, kappa, tot, nullptr, nullptr, soft, log_z, nullptr, ws, ws_bytes, strm);
  }
}

extern "C" tcq_status_t tcq_bcjr_soft_and_grad(const tcq_trellis_t *tr, const float *s,
                                               const float *D, int64_t n_seq, float temp,
                                               const float *grad_soft, float *soft,
                                               float *log_z, float *grad_s, void *ws,
                                               size_t ws_bytes, void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if (!temp_ok(temp)) return TCQ_ERR_INVALID_ARG;
  if (n_seq < 0 || n_seq > (int64_t)INT32_MAX) return TCQ_ERR_INVALID_ARG;
  if (n_seq == 0) return TCQ_OK;
  if (!s || !grad_soft || !grad_s || !aligned16(s) || !aligned16(grad_soft) || !aligned16(grad_s) ||
      (soft && !aligned16(soft)) || (log_z && !aligned16(log_z)) || (D && !aligned16(D)))
    return TCQ_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TCQ_ERR_WORKSPACE;
  const float kappa = (float)(1.4426950408889634 / (double)temp);
  const float tot = (float)(2.0 / (double)temp);
  cudaStream_t strm = (cudaStream_t)stream;
  const int T = tr->seq_len;
  switch (tr->L) {
    case 8: return launch<Grad8>(s, D, n_seq, T, kappa, tot, grad_soft, nullptr, soft, log_z, grad_s, ws, ws_bytes, strm);
    case 12: return launch<Grad12>(s, D, n_seq, T, kappa, tot, grad_soft, nullptr, soft, log_z, grad_s, ws, ws_bytes, strm);
    default: return launch<Grad16>(s, D, n_seq, T, kappa, tot, grad_soft, nullptr, soft, log_z, grad_s, ws, ws_bytes, strm);
  }
}

extern "C" tcq_status_t tcq_bcjr_soft_backward(const tcq_trellis_t *tr, const float *s,
                                               const float *D, int64_t n_seq, float temp,
                                               const float *soft,
                                               const float *grad_soft, float *grad_s, void *ws,
                                               size_t ws_bytes, void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if (!temp_ok(temp)) return TCQ_ERR_INVALID_ARG;
  if (n_seq < 0 || n_seq > (int64_t)INT32_MAX) return TCQ_ERR_INVALID_ARG;
  if (n_seq == 0) return TCQ_OK;
  if (!s || !soft || !grad_soft || !grad_s || !aligned16(s) || !aligned16(soft) ||
      !aligned16(grad_soft) || !aligned16(grad_s) || (D && !aligned16(D)))
    return TCQ_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TCQ_ERR_WORKSPACE;
  const float kappa = (float)(1.4426950408889634 / (double)temp);
  const float tot = (float)(2.0 / (double)temp);
  cudaStream_t strm = (cudaStream_t)stream;
  const int T = tr->seq_len;
  switch (tr->L) {
    case 8: return launch<Grad8>(s, D, n_seq, T, kappa, tot, grad_soft, soft, nullptr, nullptr, grad_s, ws, ws_bytes, strm);
    case 12: return launch<Grad12>(s, D, n_seq, T, kappa, tot, grad_soft, soft, nullptr, nullptr, grad_s, ws, ws_bytes, strm);
    default: return launch<Grad16>(s, D, n_seq, T, kappa, tot, grad_soft, soft, nullptr, nullptr, grad_s, ws, ws_bytes, strm);
  }
}
