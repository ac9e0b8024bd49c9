// Viterbi (min-plus) encode on the bitshift trellis, fp32, state-parallel.
//
// [QTIP blog, "The trellis: a stateful codebook"] Viterbi keeps, per step,
// the cheapest walk into each of the 2^L states; the predecessors of state j
// are computed with shifts, pred_a(j) = (j >> k) | (a << (L-k)):
//   cost_0(j) = (code_j - s_0)^2
//   cost_t(j) = min_a cost_{t-1}(pred_a j) + (code_j - s_t)^2
// and the walk is read back from the final argmin with stored backpointers.
//
// Layout used here (k = 2).  The four states j = 4q + b (b = 0..3) share the
// same predecessor set {q | a << (L-2)}, so the minimum over a, and its
// argmin, is taken once per group q: the kernel carries
//   M_t(q) = min_a cost_{t-1}(q | a << (L-2)),   M_0 = 0,
// (2^(L-2) values, a quarter of the cost vector) and recomputes
//   cost_t(p) = M_t(p >> 2) + (code_p - s_t)^2
// on the fly.  Every fp32 operation is the same correctly rounded operation
// as in the definition (sub, mul, add; no FMA contraction), so costs, paths
// and the MSE are bit-identical to a plain fp32 evaluation, and the
// backpointer needs 2 bits per GROUP per step, not per state.
//
// Work split: a sequence's 2^(L-2) groups are spread over TPS threads, G
// consecutive groups per thread.  The thread's 4G predecessor states
// p = a*2^(L-2) + G*w + i never change, so their code values are computed
// once (1MAD in registers; for L = 16 in tensor memory, because 2^16 fp32
// values are the whole register file) and the state vector M lives in shared
// memory.  Step t reads M_{t-1} at a*2^(L-4) + (G/4)*w + (0..G/4-1)
// (four short runs), writes M_t at G*w + (0..G-1) (one run) and stores the
// thread's 2G backpointer bits with one coalesced store.
#include <algorithm>

#include "tcq_device.cuh"

namespace tcq {

template <int L_, int G_, int SPC_, int AREG_, int NBUF_, int MINB_ = 1, bool TMEMC_ = false>
struct VitCfg {
  static constexpr int L = L_, G = G_, SPC = SPC_, AREG = AREG_, NBUF = NBUF_;
  static constexpr int MINB = MINB_;                // CTAs per SM the registers must allow
  static constexpr int NG = 1 << (L - 2);      // groups (states / 4)
  static constexpr int TPS = NG / G;           // threads per sequence
  static constexpr int NT = TPS * SPC;         // threads per CTA
  static constexpr int GQ = G / 4;             // M values read per predecessor digit
  static constexpr int ASM = 4 - AREG;         // predecessor digits whose codes sit in smem
  static constexpr int BPB = G / 4;            // backpointer bytes per thread per step
  static constexpr int SWZ = (GQ >= 8 ? 7 : GQ - 1);
  // several sequences per warp (L = 8: 16 threads each): a sequence steps on
  // a warp barrier, since its threads exchange values only with each other
  static constexpr bool WARPSEQ = SPC > 1 && TPS < 32 && 32 % TPS == 0;
  // the ASM digits not in registers sit in tensor memory (TMEMC: this thread's
  // lane, columns (q ASM + a - AREG) 4 + r) or in shared memory
  static constexpr bool TMEMC = TMEMC_;
  static constexpr int TCPT = TMEMC ? ASM * G : 0;                 // TMEM columns per thread
  static constexpr int TCOLS = TCPT * (NT / 128) <= 32 ? 32 : TCPT * (NT / 128);
  // MARGIN (the decision-margin pass) also stages the walk: SPC x 256 uint16
  static constexpr size_t smem_bytes(bool margin = false) {
    return sizeof(float) * ((size_t)SPC * NBUF * NG + (TMEMC ? 0 : (size_t)ASM * G * TPS) +
                            (size_t)SPC * 512) +
           sizeof(unsigned long long) * NT + (margin ? sizeof(uint16_t) * (size_t)SPC * 256 : 0);
  }
  static_assert(NG % G == 0 && G % 4 == 0, "bad group split");
  static_assert(!TMEMC || (SPC == 1 && NT % 128 == 0 && ASM % 2 == 0 && ASM > 0 &&
                           (TCOLS & (TCOLS - 1)) == 0 && TCOLS <= 512), "tensor-memory code layout");
};

template <int N>
__device__ __forceinline__ void load_run(const float *base, int idx, float *dst) {
  // N contiguous floats starting at idx (N in {1,2,4,8}; idx aligned to min(N,4))
  if constexpr (N == 1) {
    dst[0] = base[idx];
  } else if constexpr (N == 2) {
    const float2 v = *reinterpret_cast<const float2 *>(base + idx);
    dst[0] = v.x; dst[1] = v.y;
  } else {
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
      const float4 v = *reinterpret_cast<const float4 *>(base + idx + 4 * q);
      dst[4 * q] = v.x; dst[4 * q + 1] = v.y; dst[4 * q + 2] = v.z; dst[4 * q + 3] = v.w;
    }
  }
}

// Relative gap of a decision, (second - best) / max(best, 1e-30), each
// operation rounded to fp32 (costs are >= 0).
__device__ __forceinline__ float decision_gap(float best, float second) {
  return __fdiv_rn(__fsub_rn(second, best), fmaxf(best, 1e-30f));
}

// Fold candidate v into (best, second distinct above best).
__device__ __forceinline__ void fold_second(float v, float &b, float &s2) {
  if (v < b) { s2 = b; b = v; }
  else if (v > b) s2 = fminf(s2, v);
}

// MARGIN = false: the forward recursion, backpointers, final argmin and MSE.
// MARGIN = true (decision-margin pass, run after the traceback on the same
// inputs): the same recursion with no backpointers or outputs except
// margin_out[seq], the smallest relative decision margin along the walk in
// `states` -- at step t the gap between the best and second-best distinct
// cost_{t-1} over the four predecessors of states[t] (one thread per step
// reads them from the cost vector in shared memory), and at the end the gap
// between the two smallest distinct final costs.
template <class C, bool WEIGHTED, bool MARGIN = false>
__global__ void __launch_bounds__(C::NT, C::MINB)
viterbi_fwd_kernel(const float *__restrict__ s, const float *__restrict__ Dw, int64_t n_seq,
                   int T, int rot, const uint16_t *pin_states, int pin_pos,
                   uint8_t *__restrict__ bp, uint16_t *states, float *__restrict__ mse,
                   float *__restrict__ margin_out) {
  static_assert(!MARGIN || (C::NBUF == 2 && C::SPC <= 8), "margin pass: double buffer, <= 8 sequences");
  constexpr int NG = C::NG, G = C::G, GQ = C::GQ, TPS = C::TPS, AREG = C::AREG, ASM = C::ASM;
  constexpr int NB = C::NBUF;
  extern __shared__ __align__(16) float smem[];
  float *Mall = smem;                                              // [SPC][NB][NG]
  float *Csm = Mall + C::SPC * NB * NG;                            // [ASM][G/4][TPS] float4
  float *ssm = Csm + (C::TMEMC ? 0 : ASM * G * TPS);              // [SPC][256]
  float *dsm = ssm + C::SPC * 256;                                 // [SPC][256] weights
  unsigned long long *red = reinterpret_cast<unsigned long long *>(dsm + C::SPC * 256);
  uint16_t *wsm = reinterpret_cast<uint16_t *>(red + C::NT);         // MARGIN: [SPC][256] walk
  __shared__ int smg[MARGIN ? C::SPC : 1];                            // MARGIN: min step gap (bits)

  const int tid = threadIdx.x;
  const int ls = tid / TPS, w = tid - ls * TPS;
  const int64_t seq = (int64_t)blockIdx.x * C::SPC + ls;
  const bool active = seq < n_seq;

  // Code values of this thread's predecessor states p = a*NG + G*w + i, as
  // packed pairs (i, i+1).
  f2_t creg[AREG > 0 ? AREG : 1][G / 2];
#pragma unroll
  for (int a = 0; a < AREG; ++a)
#pragma unroll
    for (int i = 0; i < G; i += 2)
      creg[a][i / 2] = f2(one_mad_f32((uint32_t)(a * NG + G * w + i)),
                          one_mad_f32((uint32_t)(a * NG + G * w + i + 1)));
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
    for (int q = 0; q < GQ; ++q)
      for (int a = 0; a < ASM; a += 2) {
        const uint32_t p = (uint32_t)((a + AREG) * NG + G * w + 4 * q);
        float v[8];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          v[r] = one_mad_f32(p + r);
          v[4 + r] = one_mad_f32(p + NG + r);
        }
        tmem_st8(taddr + (uint32_t)((q * ASM + a) * 4), v);
      }
    tmem_wait_st();
  } else if (ls == 0) {
#pragma unroll
    for (int a = 0; a < ASM; ++a)
#pragma unroll
      for (int q = 0; q < GQ; ++q) {
        const uint32_t p = (uint32_t)((a + AREG) * NG + G * w + 4 * q);
        float4 v = make_float4(one_mad_f32(p), one_mad_f32(p + 1), one_mad_f32(p + 2),
                               one_mad_f32(p + 3));
        reinterpret_cast<float4 *>(Csm)[(a * GQ + q) * TPS + w] = v;
      }
  }
  // code values of digits AREG.. at group block q, from tensor or shared memory
  auto load_csm = [&](int q, float4 (&csm)[ASM > 0 ? ASM : 1]) {
    if constexpr (C::TMEMC && ASM == 4) {
      // the block's four digits are 16 consecutive columns: one load, one wait
      // (L = 16 block of 4,096 sequences: 11.99 -> 11.91 ms)
      float r16[16];
      tmem_ld16(taddr + (uint32_t)(q * ASM * 4), r16);
      tmem_wait_ld();
#pragma unroll
      for (int a = 0; a < 4; ++a)
        csm[a & (ASM > 0 ? ASM - 1 : 0)] = make_float4(r16[4 * a], r16[4 * a + 1], r16[4 * a + 2], r16[4 * a + 3]);
    } else if constexpr (C::TMEMC) {
#pragma unroll
      for (int a = 0; a < ASM; a += 2) {
        float r8[8];
        tmem_ld8(taddr + (uint32_t)((q * ASM + a) * 4), r8);
        tmem_wait_ld();
        csm[a] = make_float4(r8[0], r8[1], r8[2], r8[3]);
        csm[a + 1 < ASM ? a + 1 : 0] = a + 1 < ASM ? make_float4(r8[4], r8[5], r8[6], r8[7]) : csm[0];
      }
    } else {
#pragma unroll
      for (int a = 0; a < ASM; ++a) csm[a] = reinterpret_cast<const float4 *>(Csm)[(a * GQ + q) * TPS + w];
    }
  };
  // targets (and weights) of step t are element (t + rot) mod T of the row
  for (int x = tid; x < C::SPC * T; x += C::NT) {
    const int l = x / T, t = x - l * T;
    const int64_t sq = (int64_t)blockIdx.x * C::SPC + l;
    int tr = t + rot;
    if (tr >= T) tr -= T;
    ssm[l * 256 + t] = sq < n_seq ? s[sq * T + tr] : 0.0f;
    if (WEIGHTED) dsm[l * 256 + t] = sq < n_seq ? Dw[sq * T + tr] : 0.0f;
    if (MARGIN) wsm[l * 256 + t] = sq < n_seq ? states[sq * T + t] : (uint16_t)0;
  }
  if (MARGIN && tid < C::SPC) smg[tid] = 0x7f800000;                 // +inf
  // Pinned (tail-biting) run: the first state's top L-2 bits and the last
  // state's low L-2 bits must both equal the overlap o, i.e. only group o may
  // start (M_0 = 0 there, +inf elsewhere) and only states with low bits o may
  // end the walk.
  const int o = (pin_states != nullptr && active) ? (int)(pin_states[seq * T + pin_pos] >> 2) : -1;
  float *M = Mall + ls * NB * NG;
  for (int x = w; x < NG; x += TPS) M[swz<C::SWZ>(x)] = (o < 0 || x == o) ? 0.0f : INFINITY;
  __syncthreads();

  uint8_t *bps = bp + (active ? seq : 0) * (int64_t)(T - 1) * (NG / 4);
  float min_in[4][GQ];

  // LAZY (L = 16: double buffer, tensor-memory codes): M_{t-1} is read block
  // by block inside the step, so its 4G values are not all held in registers
  // at once (12.96 -> 11.99 ms on the 4,096-sequence block), and the final
  // decision's inputs are read after the loop
  constexpr bool LAZY = C::TMEMC && NB == 2 && GQ % 4 == 0;
  for (int t = 1; t <= (LAZY ? T - 1 : T); ++t) {
    // t < T: step computing M_t from M_{t-1}; t == T: final argmin over cost_{T-1}
    const float *Mi = M + ((t - 1) % NB) * NG;
#pragma unroll
    for (int a = 0; a < (LAZY ? 0 : 4); ++a) {
      const int base = a * (NG / 4) + GQ * w;
      if constexpr (GQ <= 4) {
        float tmp[GQ];
        load_run<GQ>(Mi, swz<C::SWZ>(base), tmp);
#pragma unroll
        for (int k = 0; k < GQ; ++k) min_in[a][k] = tmp[k];
      } else {
#pragma unroll
        for (int q = 0; q < GQ / 4; ++q) {
          float tmp[4];
          load_run<4>(Mi, swz<C::SWZ>(base + 4 * q), tmp);
#pragma unroll
          for (int k = 0; k < 4; ++k) min_in[a][4 * q + k] = tmp[k];
        }
      }
    }
    const float sv = ssm[ls * 256 + t - 1];
    if (t == T) break;
    if (NB == 1) __syncthreads();                                 // all reads of M_{t-1} done
    float *Mo = M + (t % NB) * NG;
    uint32_t bits[(2 * G + 31) / 32];
#pragma unroll
    for (int b = 0; b < (2 * G + 31) / 32; ++b) bits[b] = 0;
    // Two neighbouring groups i, i+1 with the same predecessor digit a share
    // the input M(q), so their candidate costs are computed as a packed pair:
    // d = c - s, e = d*d (written fma(d, d, +0)), cost = M + e, each lane
    // rounded exactly like the scalar operation.  A packed multiply followed
    // by the packed add is fused into one fused multiply-add by the compiler
    // (one rounding instead of two): written as a multiply, the MSE moved by
    // an ulp against the oracle's separately rounded operations.
    const f2_t sv2 = f2(sv, sv);
    const float dv = WEIGHTED ? dsm[ls * 256 + t - 1] : 1.0f;
    const f2_t dv2 = f2(dv, dv);
#pragma unroll
    for (int q = 0; q < GQ; ++q) {
      if (LAZY && (q & 3) == 0) {
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          float tmp[4];
          load_run<4>(Mi, swz<C::SWZ>(a * (NG / 4) + GQ * w + q), tmp);
#pragma unroll
          for (int k = 0; k < 4; ++k) min_in[a][(q + k) % GQ] = tmp[k];
        }
      }
      float4 csm[ASM > 0 ? ASM : 1];
      if constexpr (ASM > 0) load_csm(q, csm);
      float outv[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float clo[4], chi[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          f2_t cp;
          if (a < AREG) cp = creg[a < AREG ? a : 0][2 * q + h];
          else {
            const float4 v = csm[a >= AREG ? a - AREG : 0];
            cp = h == 0 ? f2(v.x, v.y) : f2(v.z, v.w);
          }
          const f2_t d = f2sub(cp, sv2);
          f2_t e = f2fma(d, d, 0ull);                     // RN(d*d)
          if (WEIGHTED) e = f2fma(e, dv2, 0ull);          // RN(e*D), D >= 0
          const f2_t cost = f2add(f2(min_in[a][q], min_in[a][q]), e);
          clo[a] = f2lo(cost);
          chi[a] = f2hi(cost);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float *cst = u == 0 ? clo : chi;
          const int r = 2 * h + u, i = 4 * q + r;
          // First minimum (lowest a) of the four candidates with the DPX
          // min-with-predicate: costs are sums of squares (>= +0), so their bit
          // patterns order like their values, and (x <= y) keeps the lower
          // index on ties.
          bool q1, q2, q3;
          const int m01 = __vibmin_s32(__float_as_int(cst[0]), __float_as_int(cst[1]), &q1);
          const int m23 = __vibmin_s32(__float_as_int(cst[2]), __float_as_int(cst[3]), &q2);
          const int m = __vibmin_s32(m01, m23, &q3);
          outv[r] = __int_as_float(m);
          const uint32_t idx = q3 ? (q1 ? 0u : 1u) : (q2 ? 2u : 3u);
          bits[i >> 4] |= idx << (2 * (i & 15));
        }
      }
      *reinterpret_cast<float4 *>(Mo + swz<C::SWZ>(G * w + 4 * q)) =
          make_float4(outv[0], outv[1], outv[2], outv[3]);
    }
    if constexpr (MARGIN) {
      // the walk's decision at step t: its state's four predecessors p, with
      // cost_{t-1}(p) = M_{t-1}(p >> 2) + e_{t-1}(p), rounded as in the step
      if (active && t % TPS == w) {
        const uint32_t q = wsm[ls * 256 + t] >> 2;
        float b = INFINITY, s2 = INFINITY;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const uint32_t p = q | ((uint32_t)a << (C::L - 2));
          const float d = __fsub_rn(one_mad_f32(p), sv);
          float e = __fmul_rn(d, d);
          if (WEIGHTED) e = __fmul_rn(e, dv);
          fold_second(__fadd_rn(Mi[swz<C::SWZ>((int)(p >> 2))], e), b, s2);
        }
        if (s2 < INFINITY) atomicMin(&smg[ls], __float_as_int(decision_gap(b, s2)));
      }
    } else if (active) {
      uint8_t *dst = bps + (int64_t)(t - 1) * (NG / 4) + w * C::BPB;
      if constexpr (C::BPB == 1) *dst = (uint8_t)bits[0];
      else if constexpr (C::BPB == 2) *reinterpret_cast<uint16_t *>(dst) = (uint16_t)bits[0];
      else if constexpr (C::BPB == 4) *reinterpret_cast<uint32_t *>(dst) = bits[0];
      else *reinterpret_cast<uint2 *>(dst) = make_uint2(bits[0], bits[1]);
    }
    if constexpr (C::WARPSEQ) __syncwarp();                       // M_t is this sequence's own
    else __syncthreads();
  }

  // Final decision: cost_{T-1}(p) = M_{T-1}(p >> 2) + e_{T-1}(p); lowest p wins ties.
  if constexpr (LAZY) {
    const float *Mi = M + ((T - 1) % NB) * NG;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int q = 0; q < GQ; q += 4) {
        float tmp[4];
        load_run<4>(Mi, swz<C::SWZ>(a * (NG / 4) + GQ * w + q), tmp);
#pragma unroll
        for (int k = 0; k < 4; ++k) min_in[a][q + k] = tmp[k];
      }
  }
  {
    const float sv = ssm[ls * 256 + T - 1];
    unsigned long long best = ~0ull;
    float fb = INFINITY, fs = INFINITY;                                // MARGIN: best, second
#pragma unroll
    for (int q = 0; q < GQ; ++q) {
      float4 csm[ASM > 0 ? ASM : 1];
      if constexpr (ASM > 0) load_csm(q, csm);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = 4 * q + r;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          float c;
          if (a < AREG) {
            const f2_t cp = creg[a < AREG ? a : 0][i >> 1];
            c = (i & 1) ? f2hi(cp) : f2lo(cp);
          } else {
            const float4 v = csm[a >= AREG ? a - AREG : 0];
            c = r == 0 ? v.x : r == 1 ? v.y : r == 2 ? v.z : v.w;
          }
          const float d = __fsub_rn(c, sv);
          float e = __fmul_rn(d, d);
          if (WEIGHTED) e = __fmul_rn(e, dsm[ls * 256 + T - 1]);
          const float cost = __fadd_rn(min_in[a][q], e);
          const unsigned long long key =
              ((unsigned long long)__float_as_uint(cost) << 32) | (uint32_t)(a * NG + G * w + i);
          if constexpr (MARGIN) fold_second(cost, fb, fs);
          else if (o < 0 || G * w + i == o) best = key < best ? key : best;
        }
      }
    }
    constexpr int WL = TPS < 32 ? TPS : 32;
    if constexpr (MARGIN) {
      // (best, second distinct) over the sequence's TPS threads, then the
      // smallest gap of the walk
#pragma unroll
      for (int off = WL / 2; off > 0; off >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, fb, off);
        const float os = __shfl_xor_sync(0xffffffffu, fs, off);
        fold_second(ob, fb, fs);
        fs = fminf(fs, os);
      }
      red[tid] = ((unsigned long long)__float_as_uint(fs) << 32) | __float_as_uint(fb);
      __syncthreads();
      if (w == 0 && active) {
        for (int x = WL; x < TPS; x += WL) {
          const unsigned long long v = red[tid + x];
          fold_second(__uint_as_float((uint32_t)v), fb, fs);
          fs = fminf(fs, __uint_as_float((uint32_t)(v >> 32)));
        }
        float m = __int_as_float(smg[ls]);
        if (fs < INFINITY) m = fminf(m, decision_gap(fb, fs));
        margin_out[seq] = m;
      }
    } else {
      // reduce over the sequence's TPS threads
#pragma unroll
      for (int off = WL / 2; off > 0; off >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, best, off);
        best = o < best ? o : best;
      }
      red[tid] = best;
      __syncthreads();
      if (w == 0 && active) {
        for (int x = WL; x < TPS; x += WL) {
          const unsigned long long o = red[tid + x];
          best = o < best ? o : best;
        }
        const float cost = __uint_as_float((uint32_t)(best >> 32));
        states[seq * T + T - 1] = (uint16_t)(best & 0xffffffffu);
        mse[seq] = __fdiv_rn(cost, (float)T);
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

// Traceback with the sequence's backpointers staged in shared memory (L <= 12:
// at most 64 KiB per sequence): the CTA copies them with 16-byte loads, then
// one thread walks st[t-1] = (st[t] >> 2) | (bp_t(st[t] >> 2) << (L-2)) from
// shared memory and the CTA writes the walk out coalesced.
template <int L>
__global__ void __launch_bounds__(256) viterbi_traceback_staged_kernel(const uint8_t *__restrict__ bp,
                                                                       int64_t n_seq, int T,
                                                                       uint16_t *__restrict__ states) {
  constexpr int ROW = 1 << (L - 4);                       // backpointer bytes per step
  extern __shared__ __align__(16) uint8_t sbp[];          // [T-1][ROW], then [256] uint16 walk
  uint16_t *swalk = reinterpret_cast<uint16_t *>(sbp + (size_t)(T - 1) * ROW);
  const int64_t seq = blockIdx.x;
  const uint4 *src = reinterpret_cast<const uint4 *>(bp + seq * (int64_t)(T - 1) * ROW);
  const int n16 = (T - 1) * ROW / 16;
  for (int x = threadIdx.x; x < n16; x += blockDim.x) reinterpret_cast<uint4 *>(sbp)[x] = __ldg(src + x);
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t cur = states[seq * T + T - 1];
    swalk[T - 1] = (uint16_t)cur;
    for (int t = T - 1; t > 0; --t) {
      const uint32_t q = cur >> 2;
      const uint32_t a = (sbp[(t - 1) * ROW + (q >> 2)] >> (2 * (q & 3))) & 3u;
      cur = q | (a << (L - 2));
      swalk[t - 1] = (uint16_t)cur;
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T - 1; t += blockDim.x) states[seq * T + t] = swalk[t];
}

// Traceback: one thread per sequence, st[t-1] = (st[t] >> 2) | (bp_t(st[t] >> 2) << (L-2)).
template <int L>
__global__ void __launch_bounds__(128) viterbi_traceback_kernel(const uint8_t *__restrict__ bp,
                                                                int64_t n_seq, int T,
                                                                uint16_t *__restrict__ states) {
  constexpr int NG = 1 << (L - 2);
  const int64_t seq = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (seq >= n_seq) return;
  const uint8_t *b = bp + seq * (int64_t)(T - 1) * (NG / 4);
  uint16_t *st = states + seq * T;
  uint32_t cur = st[T - 1];
  for (int t = T - 1; t > 0; --t) {
    const uint32_t q = cur >> 2;
    const uint32_t a = (__ldg(b + (int64_t)(t - 1) * (NG / 4) + (q >> 2)) >> (2 * (q & 3))) & 3u;
    cur = q | (a << (L - 2));
    st[t - 1] = (uint16_t)cur;
  }
}

}  // namespace tcq

using namespace tcq;
using namespace tcq_host;

namespace {

using Vit8 = VitCfg<8, 4, 8, 4, 2>;      // 16 threads / sequence, 8 sequences / CTA
// 128 threads / sequence, 7 per SM (one wave of 1,036): 72 registers, no spill
// (8 per SM capped the registers at 64 and spilled 8 bytes per thread, reloaded
// every step: 0.2427 vs 0.2385 ms on 1,024 sequences)
using Vit12 = VitCfg<12, 8, 1, 4, 2, 7>;
// L = 16: 512 threads / sequence, one CTA per SM; all 2^16 code values in tensor
// memory (128 columns per thread), the state vector double-buffered in shared
// memory (measured: 3.39 ms against 3.65 ms with half the codes in shared
// memory and a single buffer, 1,024 sequences)
using Vit16 = VitCfg<16, 32, 1, 0, 2, 1, true>;

size_t bp_bytes_per_seq(int L, int T) { return (size_t)(T - 1) * ((size_t)1 << (L - 4)); }

template <class C, bool WEIGHTED, bool MARGIN = false>
tcq_status_t launch_fwd_w(const float *s, const float *D, int64_t n_seq, int T, uint8_t *bp,
                          uint16_t *states, float *mse, cudaStream_t stream, int rot,
                          const uint16_t *pin_states, int pin_pos, float *margin = nullptr) {
  const size_t smem = C::smem_bytes(MARGIN);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(viterbi_fwd_kernel<C, WEIGHTED, MARGIN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return TCQ_ERR_CUDA;
  }
  const int64_t blocks = (n_seq + C::SPC - 1) / C::SPC;
  viterbi_fwd_kernel<C, WEIGHTED, MARGIN><<<(unsigned)blocks, C::NT, smem, stream>>>(
      s, D, n_seq, T, rot, pin_states, pin_pos, bp, states, mse, margin);
  return launch_status();
}

// Decision-margin pass over finished walks (states holds the walks).
template <class C>
tcq_status_t launch_margin(const float *s, const float *D, int64_t n_seq, int T, uint8_t *bp,
                           uint16_t *states, float *margin, cudaStream_t stream) {
  return D ? launch_fwd_w<C, true, true>(s, D, n_seq, T, bp, states, nullptr, stream, 0, nullptr, 0,
                                         margin)
           : launch_fwd_w<C, false, true>(s, nullptr, n_seq, T, bp, states, nullptr, stream, 0,
                                          nullptr, 0, margin);
}

template <class C>
tcq_status_t launch_fwd(const float *s, int64_t n_seq, int T, uint8_t *bp, uint16_t *states,
                        float *mse, cudaStream_t stream, const float *D = nullptr, int rot = 0,
                        const uint16_t *pin_states = nullptr, int pin_pos = 0) {
  return D ? launch_fwd_w<C, true>(s, D, n_seq, T, bp, states, mse, stream, rot, pin_states, pin_pos)
           : launch_fwd_w<C, false>(s, nullptr, n_seq, T, bp, states, mse, stream, rot, pin_states,
                                    pin_pos);
}

template <int L>
tcq_status_t launch_traceback_staged(const uint8_t *bp, int64_t n_seq, int T, uint16_t *states,
                                     cudaStream_t stream) {
  const size_t smem = (size_t)(T - 1) * ((size_t)1 << (L - 4)) + 256 * sizeof(uint16_t);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(viterbi_traceback_staged_kernel<L>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return TCQ_ERR_CUDA;
  viterbi_traceback_staged_kernel<L><<<(unsigned)n_seq, 256, smem, stream>>>(bp, n_seq, T, states);
  return launch_status();
}

tcq_status_t launch_traceback(int L, const uint8_t *bp, int64_t n_seq, int T, uint16_t *states,
                              cudaStream_t stream) {
  switch (L) {
    case 8: return launch_traceback_staged<8>(bp, n_seq, T, states, stream);
    case 12: return launch_traceback_staged<12>(bp, n_seq, T, states, stream);
    default:
      viterbi_traceback_kernel<16><<<(unsigned)((n_seq + 127) / 128), 128, 0, stream>>>(bp, n_seq, T,
                                                                                        states);
      return launch_status();
  }
}

}  // namespace

extern "C" size_t tcq_viterbi_workspace_size(const tcq_trellis_t *tr, int64_t n_seq) {
  if (check_trellis(tr) != TCQ_OK || n_seq < 0) return 0;
  return ((bp_bytes_per_seq(tr->L, tr->seq_len) * (size_t)n_seq + 255) / 256) * 256 + 256;
}

extern "C" tcq_status_t tcq_viterbi_encode(const tcq_trellis_t *tr, const float *s,
                                           const float *D, int64_t n_seq, uint16_t *states,
                                           float *mse, float *min_margin, void *ws,
                                           size_t ws_bytes, void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if (n_seq < 0 || n_seq > (int64_t)INT32_MAX * 8) return TCQ_ERR_INVALID_ARG;
  if (n_seq == 0) return TCQ_OK;
  if (!s || !states || !mse || !aligned16(s) || !aligned16(states) || !aligned16(mse) ||
      (D && !aligned16(D)) || (min_margin && !aligned16(min_margin)))
    return TCQ_ERR_INVALID_ARG;
  const size_t need = tcq_viterbi_workspace_size(tr, n_seq);
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TCQ_ERR_WORKSPACE;
  const int T = tr->seq_len;
  uint8_t *bp = static_cast<uint8_t *>(ws);
  cudaStream_t strm = (cudaStream_t)stream;
  switch (tr->L) {
    case 8: st = launch_fwd<Vit8>(s, n_seq, T, bp, states, mse, strm, D); break;
    case 12: st = launch_fwd<Vit12>(s, n_seq, T, bp, states, mse, strm, D); break;
    default: st = launch_fwd<Vit16>(s, n_seq, T, bp, states, mse, strm, D); break;
  }
  if (st != TCQ_OK) return st;
  if (T > 1 && (st = launch_traceback(tr->L, bp, n_seq, T, states, strm)) != TCQ_OK) return st;
  if (!min_margin) return TCQ_OK;
  switch (tr->L) {
    case 8: return launch_margin<Vit8>(s, D, n_seq, T, bp, states, min_margin, strm);
    case 12: return launch_margin<Vit12>(s, D, n_seq, T, bp, states, min_margin, strm);
    default: return launch_margin<Vit16>(s, D, n_seq, T, bp, states, min_margin, strm);
  }
}

// Tail-biting encode [QTIP blog, "Tail-biting is worth its complexity"]: two
// runs.  First a free run on the sequence rotated by T/2, so that the wrap
// point T-1 -> 0 sits in the middle of the walk; the state that lands on
// original position 0 gives the overlap o (its top L-2 bits).  Then a run on
// the original sequence with the first state's top bits and the last state's
// low bits pinned to o: the result is a tail-biting walk whose stream is
// exactly 2*T bits.  The first run's walk is written to `states` and read
// back by the second run's prologue (stream order separates them).
template <class C>
static tcq_status_t tailbiting_passes(const float *s, const float *D, int64_t n_seq, int T,
                                      uint8_t *bp, uint16_t *states, float *mse, int L,
                                      cudaStream_t strm) {
  const int h = T / 2;
  tcq_status_t st = launch_fwd<C>(s, n_seq, T, bp, states, mse, strm, D, h);
  if (st != TCQ_OK) return st;
  if ((st = launch_traceback(L, bp, n_seq, T, states, strm)) != TCQ_OK) return st;
  st = launch_fwd<C>(s, n_seq, T, bp, states, mse, strm, D, 0, states, (T - h) % T);
  if (st != TCQ_OK) return st;
  return launch_traceback(L, bp, n_seq, T, states, strm);
}

extern "C" tcq_status_t tcq_viterbi_encode_tailbiting(const tcq_trellis_t *tr, const float *s,
                                                      const float *D, int64_t n_seq,
                                                      uint16_t *states, float *mse, void *ws,
                                                      size_t ws_bytes, void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if ((int64_t)tr->k * tr->seq_len < tr->L || tr->seq_len < 2) return TCQ_ERR_UNSUPPORTED;
  if (n_seq < 0 || n_seq > (int64_t)INT32_MAX * 8) return TCQ_ERR_INVALID_ARG;
  if (n_seq == 0) return TCQ_OK;
  if (!s || !states || !mse || !aligned16(s) || !aligned16(states) || !aligned16(mse) ||
      (D && !aligned16(D)))
    return TCQ_ERR_INVALID_ARG;
  const size_t need = tcq_viterbi_workspace_size(tr, n_seq);
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TCQ_ERR_WORKSPACE;
  uint8_t *bp = static_cast<uint8_t *>(ws);
  cudaStream_t strm = (cudaStream_t)stream;
  switch (tr->L) {
    case 8: return tailbiting_passes<Vit8>(s, D, n_seq, tr->seq_len, bp, states, mse, 8, strm);
    case 12: return tailbiting_passes<Vit12>(s, D, n_seq, tr->seq_len, bp, states, mse, 12, strm);
    default: return tailbiting_passes<Vit16>(s, D, n_seq, tr->seq_len, bp, states, mse, 16, strm);
  }
}

// ---------------------------------------------------------------------------
// Allocation-free Viterbi encode.
//
// Some callers may not allocate device memory when they call us: a plugin
// whose host owns all device memory and hands it only the inputs and outputs,
// or a deployment whose memory budget is fixed at start-up and that forbids
// cudaMalloc afterwards.  This entry point keeps the backpointers in a fixed
// buffer that is part of the library image instead of a caller workspace.
//
// The buffer below is a host-side symbol as far as host code is concerned:
// its address on the device must be fetched with cudaGetSymbolAddress, with
// the device current, before it can be passed to a kernel.  That is done once
// per device context, by the first call in it, and cached.  The cache is keyed
// on the context's unique id as well as the device ordinal: cudaDeviceReset
// destroys the device's primary context, the library's module is loaded again
// in the next one and the buffer may then sit at another address.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB per device
constexpr int kNoAllocMaxDevices = 64;

struct NoAllocSlot {
  uint8_t *ptr = nullptr;
  unsigned long long ctx_id = 0;      // unique id of the context ptr belongs to
};
NoAllocSlot g_noalloc_slot[kNoAllocMaxDevices];
std::mutex g_noalloc_mutex;

// Unique id of the calling thread's current context, through the driver entry
// points the runtime hands out (no link-time dependency on the driver
// library); false if there is no current context or the query fails.
bool current_context_id(unsigned long long *id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace

static __device__ __align__(256) uint8_t tcq_noalloc_scratch[kNoAllocScratchBytes];

static tcq_status_t noalloc_scratch_for_current_device(uint8_t **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TCQ_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return TCQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocSlot &slot = g_noalloc_slot[dev];
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  if (slot.ptr == nullptr || !have_id || id != slot.ctx_id) {
    void *addr = nullptr;          // also makes the device's primary context current
    if (cudaGetSymbolAddress(&addr, tcq_noalloc_scratch) != cudaSuccess || addr == nullptr)
      return TCQ_ERR_CUDA;
    slot.ptr = static_cast<uint8_t *>(addr);
    // the id of the context the address was looked up in (0 = unknown: the
    // next call looks it up again)
    slot.ctx_id = current_context_id(&id) ? id : 0;
  }
  *out = slot.ptr;
  return TCQ_OK;
}

extern "C" tcq_status_t tcq_viterbi_encode_noalloc(const tcq_trellis_t *tr, const float *s,
                                                   int64_t n_seq, uint16_t *states, float *mse,
                                                   void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if (n_seq < 0 || n_seq > (int64_t)INT32_MAX * 8) return TCQ_ERR_INVALID_ARG;
  if (n_seq == 0) return TCQ_OK;
  if (!s || !states || !mse || !aligned16(s) || !aligned16(states) || !aligned16(mse))
    return TCQ_ERR_INVALID_ARG;
  const int T = tr->seq_len;
  // every backpointer byte a call reads is written earlier in the same call,
  // so the buffer needs no clearing between calls
  if (bp_bytes_per_seq(tr->L, T) * (size_t)n_seq > kNoAllocScratchBytes) return TCQ_ERR_WORKSPACE;
  uint8_t *bp = nullptr;
  st = noalloc_scratch_for_current_device(&bp);
  if (st != TCQ_OK) return st;
  cudaStream_t strm = (cudaStream_t)stream;
  switch (tr->L) {
    case 8: st = launch_fwd<Vit8>(s, n_seq, T, bp, states, mse, strm); break;
    case 12: st = launch_fwd<Vit12>(s, n_seq, T, bp, states, mse, strm); break;
    default: st = launch_fwd<Vit16>(s, n_seq, T, bp, states, mse, strm); break;
  }
  if (st != TCQ_OK || T == 1) return st;
  const unsigned tb_blocks = (unsigned)((n_seq + 127) / 128);
  switch (tr->L) {
    case 8: viterbi_traceback_kernel<8><<<tb_blocks, 128, 0, strm>>>(bp, n_seq, T, states); break;
    case 12: viterbi_traceback_kernel<12><<<tb_blocks, 128, 0, strm>>>(bp, n_seq, T, states); break;
    default: viterbi_traceback_kernel<16><<<tb_blocks, 128, 0, strm>>>(bp, n_seq, T, states); break;
  }
  return launch_status();
}
