// Sliding-window decode and state packing.
//
// [QTIP blog, "The trellis: a stateful codebook"] the state of weight t is the
// L-bit window of the bitstream starting at bit k*t (most significant first),
// so every weight decodes on its own: a funnel shift, the 1MAD hash and a
// conversion to fp16.  [QTIP blog, "Tail-biting is worth its complexity"] a
// tail-biting stream is exactly k*T bits and its windows wrap around.
// [QTIP blog, "What it buys end to end"] each 16x16 tile of a weight matrix is
// one 256-weight sequence.
//
// The decode is bound by HBM traffic (2 bits in, 16 bits out per weight): the
// tile kernel keeps a sequence's 64-byte stream in registers and writes each
// tile row with one 16-byte store per thread, a warp covering 512 contiguous
// bytes of the output matrix.
#include <algorithm>

#include "tcq_device.cuh"

namespace tcq {

// Window of L bits starting at bit offset o (0..31) of the 64-bit word pair
// (hi:lo), most significant bit first.
template <int L>
__device__ __forceinline__ uint32_t window_at(uint32_t hi, uint32_t lo, uint32_t o) {
  return __funnelshift_l(lo, hi, o) >> (32 - L);
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// TILE16 decode of 256-weight sequences (k = 2, so a sequence's stream is 16
// words tail-biting, 16 + ceil((L-2)/32) words free-start).  One thread owns
// one half (8 columns) of one tile and walks its 16 rows.
template <int L, int LAYOUT>
__global__ void __launch_bounds__(256) decode_tile16_kernel(const uint32_t *__restrict__ bits,
                                                            int n_tiles_c, int64_t n_items,
                                                            int words_per_seq, int cols,
                                                            uint16_t *__restrict__ out) {
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_items;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tr = g / (2 * n_tiles_c);
    const int rem = (int)(g - tr * 2 * n_tiles_c);
    const int tc = rem >> 1, h = rem & 1;
    const int64_t seq = tr * n_tiles_c + tc;
    const uint32_t *src = bits + seq * words_per_seq;
    uint32_t w[17];
    if (LAYOUT == TCQ_TAILBITING) {
      const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v = __ldg(s4 + q);
        w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
      }
      w[16] = w[0];
    } else {
#pragma unroll
      for (int q = 0; q < 16; ++q) w[q] = __ldg(src + q);
      w[16] = __ldg(src + 16);
    }
    uint16_t *dst = out + (tr * 16) * (int64_t)cols + tc * 16 + h * 8;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      // weights t = 16 r + 8 h + j, stream bit 2t = 32 r + 16 h + 2 j
      uint32_t hv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const unsigned long long c2 =
            one_mad_decode_f32x2(window_at<L>(w[r], w[r + 1], 16 * h + 4 * j),
                                 window_at<L>(w[r], w[r + 1], 16 * h + 4 * j + 2));
        hv[j] = pack_half2(__uint_as_float((uint32_t)c2), __uint_as_float((uint32_t)(c2 >> 32)));
      }
      uint4 o;
      o.x = hv[0]; o.y = hv[1]; o.z = hv[2]; o.w = hv[3];
      *reinterpret_cast<uint4 *>(dst + (int64_t)r * cols) = o;
    }
  }
}

// Generic decode, one thread per weight, output in sequence order.
template <int L>
__global__ void __launch_bounds__(256) decode_seq_kernel(const uint32_t *__restrict__ bits,
                                                         int64_t n_weights, int T, int layout,
                                                         int words_per_seq, int nbits,
                                                         uint16_t *__restrict__ out) {
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_weights;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t seq = g / T;
    const int t = (int)(g - seq * T);
    const uint32_t *src = bits + seq * words_per_seq;
    const int p = 2 * t;              // k = 2
    const int i = p >> 5, o = p & 31;
    const uint32_t hi = __ldg(src + i);
    int i1 = i + 1;
    uint32_t lo = 0;
    if (layout == TCQ_TAILBITING) {
      if (i1 == words_per_seq) i1 = 0;
      lo = __ldg(src + i1);
    } else if (i1 < words_per_seq) {
      lo = __ldg(src + i1);
    }
    (void)nbits;
    const float c = one_mad_decode_f32(window_at<L>(hi, lo, (uint32_t)o));
    out[g] = __half_as_ushort(__float2half_rn(c));
  }
}

// Pack walks into streams: one thread per output word.
__global__ void __launch_bounds__(256) pack_states_kernel(const uint16_t *__restrict__ states,
                                                          int64_t n_words_total, int T, int L,
                                                          int layout, int words_per_seq,
                                                          uint32_t *__restrict__ bits) {
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_words_total;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t seq = g / words_per_seq;
    const int wi = (int)(g - seq * words_per_seq);
    const uint16_t *st = states + seq * T;
    const int kT = 2 * T;
    const int nbits = layout == TCQ_TAILBITING ? kT : kT + L - 2;
    uint32_t word = 0;
    for (int b = 0; b < 32; ++b) {
      const int p = 32 * wi + b;
      uint32_t bit = 0;
      if (p < kT) {
        const int t = p >> 1, i = p & 1;          // top bits of state t
        bit = (st[t] >> (L - 1 - i)) & 1u;
      } else if (p < nbits) {
        const int i = p - 2 * (T - 1);            // tail of the last state
        bit = (st[T - 1] >> (L - 1 - i)) & 1u;
      }
      word |= bit << (31 - b);
    }
    bits[g] = word;
  }
}

}  // namespace tcq

using namespace tcq;
using namespace tcq_host;

extern "C" size_t tcq_stream_words(const tcq_trellis_t *tr, int layout) {
  if (check_trellis(tr) != TCQ_OK) return 0;
  const int64_t kT = (int64_t)tr->k * tr->seq_len;
  if (layout == TCQ_TAILBITING) {
    if (kT % 32 != 0 || kT < tr->L) return 0;
    return (size_t)(kT / 32);
  }
  if (layout == TCQ_FREE_START) return (size_t)((kT + tr->L - tr->k + 31) / 32);
  return 0;
}

extern "C" tcq_status_t tcq_pack_states(const tcq_trellis_t *tr, const uint16_t *states,
                                        int64_t n_seq, int layout, uint32_t *bits,
                                        void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if (layout != TCQ_TAILBITING && layout != TCQ_FREE_START) return TCQ_ERR_INVALID_ARG;
  if (n_seq < 0) return TCQ_ERR_INVALID_ARG;
  const size_t wps = tcq_stream_words(tr, layout);
  if (wps == 0) return TCQ_ERR_UNSUPPORTED;
  if (n_seq == 0) return TCQ_OK;
  if (!states || !bits || !aligned16(states) || !aligned16(bits)) return TCQ_ERR_INVALID_ARG;
  const int64_t total = n_seq * (int64_t)wps;
  const int64_t blocks = std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 16);
  pack_states_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      states, total, tr->seq_len, tr->L, layout, (int)wps, bits);
  return launch_status();
}

template <int L>
static tcq_status_t decode_launch(const tcq_trellis_t *tr, const uint32_t *bits, int64_t n_seq,
                                  int layout, int out_layout, int64_t rows, int64_t cols,
                                  uint16_t *out, cudaStream_t stream, int wps) {
  if (out_layout == TCQ_OUT_TILE16) {
    const int64_t ntc = cols / 16;
    const int64_t items = n_seq * 2;
    // one item per thread: the block scheduler overlaps one CTA's loads with
    // another's stores better than a capped grid-stride loop (26.6 vs 28.7 us
    // on the 8192^2 matrix)
    const int64_t blocks = std::min<int64_t>((items + 255) / 256, (int64_t)INT32_MAX);
    if (layout == TCQ_TAILBITING)
      decode_tile16_kernel<L, TCQ_TAILBITING><<<(unsigned)blocks, 256, 0, stream>>>(
          bits, (int)ntc, items, wps, (int)cols, out);
    else
      decode_tile16_kernel<L, TCQ_FREE_START><<<(unsigned)blocks, 256, 0, stream>>>(
          bits, (int)ntc, items, wps, (int)cols, out);
  } else {
    const int64_t nw = n_seq * tr->seq_len;
    const int64_t blocks = std::min<int64_t>((nw + 255) / 256, (int64_t)sm_count() * 16);
    decode_seq_kernel<L><<<(unsigned)blocks, 256, 0, stream>>>(
        bits, nw, tr->seq_len, layout, wps, 0, out);
  }
  (void)rows;
  return launch_status();
}

extern "C" tcq_status_t tcq_decode(const tcq_trellis_t *tr, const uint32_t *bits, int64_t n_seq,
                                   int layout, int out_layout, int64_t rows, int64_t cols,
                                   uint16_t *out, void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if (layout != TCQ_TAILBITING && layout != TCQ_FREE_START) return TCQ_ERR_INVALID_ARG;
  if (out_layout != TCQ_OUT_SEQ && out_layout != TCQ_OUT_TILE16) return TCQ_ERR_INVALID_ARG;
  if (n_seq < 0) return TCQ_ERR_INVALID_ARG;
  const size_t wps = tcq_stream_words(tr, layout);
  if (wps == 0) return TCQ_ERR_UNSUPPORTED;
  if (out_layout == TCQ_OUT_TILE16) {
    if (tr->seq_len != 256) return TCQ_ERR_UNSUPPORTED;
    if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16) return TCQ_ERR_INVALID_ARG;
    if ((rows / 16) * (cols / 16) != n_seq) return TCQ_ERR_INVALID_ARG;
    if (cols > (int64_t)INT32_MAX / 2 || rows / 16 > (int64_t)INT32_MAX) return TCQ_ERR_UNSUPPORTED;
  }
  if (n_seq == 0) return TCQ_OK;
  if (!bits || !out || !aligned16(bits) || !aligned16(out)) return TCQ_ERR_INVALID_ARG;
  if (out_layout == TCQ_OUT_TILE16 && layout == TCQ_FREE_START && wps > 17) return TCQ_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  switch (tr->L) {
    case 8: return decode_launch<8>(tr, bits, n_seq, layout, out_layout, rows, cols, out, s, (int)wps);
    case 12: return decode_launch<12>(tr, bits, n_seq, layout, out_layout, rows, cols, out, s, (int)wps);
    default: return decode_launch<16>(tr, bits, n_seq, layout, out_layout, rows, cols, out, s, (int)wps);
  }
}

// ---------------------------------------------------------------------------
// Decode fused into a matrix-vector product [QTIP blog, "What it buys end to
// end": each 16x16 tile is one 256-weight sequence that decodes straight into
// the matmul operand, so the weights never exist in memory at 16 bits].
//   y[i] = sum_j W[i][j] x[j],  W = the fp16 matrix tcq_decode (TILE16) gives,
// accumulated in fp32.  A warp takes a run of tile-columns along two
// tile-rows; each lane owns one row of one of them and decodes that row's 16
// weights in every tile of the run and multiplies them by x; the stream words
// of the next tile are loaded while the current one decodes.  Runs combine by
// one fp32 atomic add per row into y (zeroed first on the same stream).
//
// The fp16 code of a weight depends only on the byte sum of its LCG output
// (1,021 values), so each CTA first fills a shared-memory table of the 1,021
// fp16 codes (held as fp32, the value the product multiplies), one copy per
// lane: entry (bs, lane) at float index 32 bs + lane, so a warp's 32 lookups
// fall in 32 different banks whatever the byte sums are.  One IDP4A with byte
// weights 128 and accumulator 4 lane gives the entry's byte offset straight
// from the LCG output.  Products are paired per lane (even and odd weights of
// the row) and summed in fp32.  One 1024-thread CTA per SM (the table takes
// 130,688 bytes).  Measured and not kept: x staged in shared memory beside the
// table (2.1 M more warp instructions, 2 us slower on 8192 x 8192).
namespace tcq {

constexpr int kGemvLutRows = 1021;

template <int L, int LAYOUT>
__global__ void __launch_bounds__(1024, 1) decode_gemv_lut_kernel(const uint32_t *__restrict__ bits,
                                                                  int n_tr, int n_tc, int runs, int wps,
                                                                  const float *__restrict__ x,
                                                                  float *__restrict__ y) {
  extern __shared__ __align__(16) float lut[];           // [1021][32]
  const int lane = threadIdx.x & 31;
  // thread e computes entry e once and stores its 32 copies as eight 16-byte
  // chunks, starting at chunk (lane mod 8) so that a warp's stores spread over
  // all banks
  for (int e = threadIdx.x; e < kGemvLutRows; e += blockDim.x) {
    const float v = __half2float(__float2half_rn(__fmul_rn((float)(e - 510), 0x1.bb68f6p-8f)));
    float4 *dst = reinterpret_cast<float4 *>(lut + e * 32);
#pragma unroll
    for (int q = 0; q < 8; ++q) dst[(q + lane) & 7] = make_float4(v, v, v, v);
  }
  __syncthreads();
  const int r = lane & 15, half = lane >> 4;
  const uint32_t lane_off = 4u * (uint32_t)lane;
  const char *lut_b = reinterpret_cast<const char *>(lut);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int n_pairs = (n_tr + 1) >> 1;
  const int per_run = (n_tc + runs - 1) / runs;
  for (int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       wid < (int64_t)n_pairs * runs; wid += warps) {
    const int pair = (int)(wid / runs), run = (int)(wid - (int64_t)pair * runs);
    const int tr = min(2 * pair + half, n_tr - 1);
    const bool owner = 2 * pair + half < n_tr;
    const int c0 = run * per_run, c1 = min(n_tc, c0 + per_run);
    if (c0 >= c1) continue;
    const uint32_t *row_src = bits + (int64_t)tr * n_tc * wps + r;
    const int r1 = LAYOUT == TCQ_TAILBITING ? (((r + 1) & 15) - r) : 1;   // offset of word r+1
    uint32_t nw0 = __ldg(row_src + (int64_t)c0 * wps), nw1 = __ldg(row_src + (int64_t)c0 * wps + r1);
    f2_t acc = f2(0.0f, 0.0f);
    for (int tc = c0; tc < c1; ++tc) {
      const uint32_t w0 = nw0, w1 = nw1;
      if (tc + 1 < c1) {                               // next tile's words, one tile ahead
        nw0 = __ldg(row_src + (int64_t)(tc + 1) * wps);
        nw1 = __ldg(row_src + (int64_t)(tc + 1) * wps + r1);
      }
      const float4 *xq = reinterpret_cast<const float4 *>(x + tc * 16);
      const float4 x0 = __ldg(xq), x1 = __ldg(xq + 1), x2 = __ldg(xq + 2), x3 = __ldg(xq + 3);
      const float xv[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                            x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {                    // weights 2j, 2j+1 of the row
        const uint32_t s0 = window_at<L>(w0, w1, 4 * j) * kLcgMul + kLcgAdd;
        const uint32_t s1 = window_at<L>(w0, w1, 4 * j + 2) * kLcgMul + kLcgAdd;
        const float v0 = *reinterpret_cast<const float *>(lut_b + __dp4a(s0, 0x80808080u, lane_off));
        const float v1 = *reinterpret_cast<const float *>(lut_b + __dp4a(s1, 0x80808080u, lane_off));
        acc = f2fma(f2(v0, v1), f2(xv[2 * j], xv[2 * j + 1]), acc);
      }
    }
    if (owner) atomicAdd(y + (int64_t)tr * 16 + r, f2lo(acc) + f2hi(acc));
  }
}

template <int L, int LAYOUT>
tcq_status_t gemv_launch(const uint32_t *bits, int n_tr, int n_tc, int wps, const float *x, float *y,
                         cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)kGemvLutRows * 32;
  if (cudaFuncSetAttribute(decode_gemv_lut_kernel<L, LAYOUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return TCQ_ERR_CUDA;
  // each warp a run of tiles along a tile-row pair, runs per pair chosen so
  // that every resident warp has work
  const int64_t n_pairs = (n_tr + 1) / 2;
  const int64_t resident_warps = (int64_t)sm_count() * 32;
  const int runs = (int)std::max<int64_t>(1, std::min<int64_t>(n_tc, resident_warps / n_pairs));
  const int64_t warps = n_pairs * runs;
  const unsigned blocks = (unsigned)std::min<int64_t>((warps + 31) / 32, (int64_t)sm_count());
  decode_gemv_lut_kernel<L, LAYOUT><<<blocks, 1024, smem, s>>>(bits, n_tr, n_tc, runs, wps, x, y);
  return launch_status();
}

}  // namespace tcq

extern "C" tcq_status_t tcq_decode_gemv(const tcq_trellis_t *tr, const uint32_t *bits, int layout,
                                        int64_t rows, int64_t cols, const float *x, float *y,
                                        void *stream) {
  tcq_status_t st = check_trellis(tr);
  if (st != TCQ_OK) return st;
  if (layout != TCQ_TAILBITING && layout != TCQ_FREE_START) return TCQ_ERR_INVALID_ARG;
  if (tr->seq_len != 256) return TCQ_ERR_UNSUPPORTED;
  if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16) return TCQ_ERR_INVALID_ARG;
  if (rows / 16 > INT32_MAX || cols / 16 > INT32_MAX) return TCQ_ERR_UNSUPPORTED;
  const size_t wps = tcq_stream_words(tr, layout);
  if (wps == 0 || wps > 17) return TCQ_ERR_UNSUPPORTED;
  if (!bits || !x || !y || !aligned16(bits) || !aligned16(x) || !aligned16(y))
    return TCQ_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(y, 0, sizeof(float) * (size_t)rows, s) != cudaSuccess) return TCQ_ERR_CUDA;
  const int n_tr = (int)(rows / 16), n_tc = (int)(cols / 16);
  const bool tb = layout == TCQ_TAILBITING;
  switch (tr->L) {
    case 8: return tb ? gemv_launch<8, TCQ_TAILBITING>(bits, n_tr, n_tc, (int)wps, x, y, s)
                      : gemv_launch<8, TCQ_FREE_START>(bits, n_tr, n_tc, (int)wps, x, y, s);
    case 12: return tb ? gemv_launch<12, TCQ_TAILBITING>(bits, n_tr, n_tc, (int)wps, x, y, s)
                       : gemv_launch<12, TCQ_FREE_START>(bits, n_tr, n_tc, (int)wps, x, y, s);
    default: return tb ? gemv_launch<16, TCQ_TAILBITING>(bits, n_tr, n_tc, (int)wps, x, y, s)
                       : gemv_launch<16, TCQ_FREE_START>(bits, n_tr, n_tc, (int)wps, x, y, s);
  }
}
