// Random-sign Hadamard rotation of a weight matrix.
//
// [QTIP blog, "The trellis: a stateful codebook"] before quantisation QuIP#'s
// transform is applied from the left and the right, +-1 signs followed by a
// Hadamard transform, so that the entries end up close to i.i.d. Gaussian:
//   out = (H_R / sqrt R) diag(sign_rows) W diag(sign_cols) (H_C / sqrt C),
// H_n the Sylvester Hadamard matrix.  The product is separable, so it runs as
// fast Walsh-Hadamard butterflies, (a, b) -> (a + b, a - b):
//   * row pass: one CTA per row.  For 2^11 <= C <= 2^13 the row lives in
//     registers (log2(C/256) levels), crosses shared memory once and finishes
//     in registers and lane shuffles; narrower rows go through shared memory
//     (the first two levels in registers on the 16-byte load, then radix-4
//     levels).  Row sign and 1/sqrt C on the store;
//   * column passes: tiles of 32 columns (128-byte row segments) by the
//     2^nb rows that differ only in one chunk of nb row-index bits; the chunks
//     together cover log2(R) bits; in place; the last chunk scales by
//     1/sqrt R.  For 2^12 <= R <= 2^24 the chunks are 6..8 bits and run in
//     registers around one shared-memory transpose; otherwise chunks of up
//     to 10 bits run as radix-4 levels in shared memory.
// Bound by HBM traffic: 8 bytes per element per pass (one row pass and
// ceil(log2 R / 10) column passes).
#include <algorithm>

#include "tcq_device.cuh"

namespace tcq {

__global__ void __launch_bounds__(256) rht_rows_kernel(const float *__restrict__ W, int R, int C,
                                                       const float *__restrict__ sign_rows,
                                                       const float *__restrict__ sign_cols,
                                                       float scale, float *out) {
  extern __shared__ __align__(16) float xs[];   // [C]
  int lc = 0;
  while ((1 << lc) < C) ++lc;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    const float4 *src = reinterpret_cast<const float4 *>(W + (int64_t)r * C);
    const float4 *sg = reinterpret_cast<const float4 *>(sign_cols);
    for (int q = threadIdx.x; q < C / 4; q += blockDim.x) {
      const float4 v = src[q], g = __ldg(sg + q);
      const float x0 = v.x * g.x, x1 = v.y * g.y, x2 = v.z * g.z, x3 = v.w * g.w;
      const float a0 = x0 + x1, a1 = x0 - x1, a2 = x2 + x3, a3 = x2 - x3;   // level h = 1
      reinterpret_cast<float4 *>(xs)[q] = make_float4(a0 + a2, a1 + a3, a0 - a2, a1 - a3);  // h = 2
    }
    __syncthreads();
    // remaining levels two at a time: radix-4 butterflies on i, i+h, i+2h, i+3h
    int lh = 2;
    for (; lh + 2 <= lc; lh += 2) {
      const int h = 1 << lh;
      for (int p = threadIdx.x; p < C / 4; p += blockDim.x) {
        const int i = ((p >> lh) << (lh + 2)) | (p & (h - 1));
        const float x0 = xs[i], x1 = xs[i + h], x2 = xs[i + 2 * h], x3 = xs[i + 3 * h];
        const float a0 = x0 + x1, a1 = x0 - x1, a2 = x2 + x3, a3 = x2 - x3;
        xs[i] = a0 + a2; xs[i + h] = a1 + a3; xs[i + 2 * h] = a0 - a2; xs[i + 3 * h] = a1 - a3;
      }
      __syncthreads();
    }
    if (lh < lc) {                                      // one level left
      const int h = 1 << lh;
      for (int p = threadIdx.x; p < C / 2; p += blockDim.x) {
        const int i = ((p >> lh) << (lh + 1)) | (p & (h - 1));
        const float a = xs[i], b = xs[i + h];
        xs[i] = a + b;
        xs[i + h] = a - b;
      }
      __syncthreads();
    }
    const float f = sign_rows[r] * scale;
    float4 *dst = reinterpret_cast<float4 *>(out + (int64_t)r * C);
    for (int q = threadIdx.x; q < C / 4; q += blockDim.x) {
      const float4 v = reinterpret_cast<const float4 *>(xs)[q];
      dst[q] = make_float4(v.x * f, v.y * f, v.z * f, v.w * f);
    }
    __syncthreads();
  }
}

// Row pass for C = 2^LC, 2^11 <= C <= 2^13, with one shared-memory round trip
// per row.  Index j = a*256 + t (t < 256, a < E = C/256):
//   stage 1: thread t loads x[a*256 + t] for all a (coalesced), applies the
//            column signs and runs the log2(E) butterfly levels over a in
//            registers, then stores to shared memory;
//   stage 2: thread (group a, m < P = 256/E) reads the E consecutive values
//            a*256 + m*E .. + E-1 and runs log2(E) levels in registers;
//   stage 3: the last log2(P) levels: for E >= 16 after a second pass through
//            shared memory, in registers, with coalesced stores; for E = 8
//            across the P lanes of a group with shuffles.  Row sign and
//            1/sqrt C on the store.
// Shared memory holds the row with 4 floats of padding per 32, which keeps
// both the stage-1 stores and the stage-2 vector loads bank-conflict free.
template <int LC>
__global__ void __launch_bounds__(256, LC == 13 ? 3 : 4) rht_rows_reg_kernel(const float *W, int R,
                                                           const float *__restrict__ sign_rows,
                                                           const float *__restrict__ sign_cols,
                                                           float scale, float *out) {
  constexpr int C = 1 << LC, E = C / 256, P = 256 / E;
  __shared__ __align__(16) float xs[C + C / 8];
  const int t = threadIdx.x;
  const int ga = t / P, m = t - ga * P;                   // stage-2 group and rank in it
  uint32_t neg = 0;                                       // bit a: sign_cols[a*256 + t] < 0
#pragma unroll
  for (int a = 0; a < E; ++a) neg |= (__ldg(sign_cols + a * 256 + t) < 0.0f ? 1u : 0u) << a;
  auto pad = [](int idx) { return idx + (idx >> 5) * 4; };
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    const float *src = W + (int64_t)r * C;
    float v[E];
#pragma unroll
    for (int a = 0; a < E; ++a)
      v[a] = __uint_as_float(__float_as_uint(src[a * 256 + t]) ^ (((neg >> a) & 1u) << 31));
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
      for (int i = 0; i < E; ++i)
        if ((i & h) == 0) {
          const float x = v[i], y = v[i + h];
          v[i] = x + y;
          v[i + h] = x - y;
        }
#pragma unroll
    for (int a = 0; a < E; ++a) xs[pad(a * 256 + t)] = v[a];
    __syncthreads();
    const int base = ga * 256 + m * E;
#pragma unroll
    for (int q = 0; q < E / 4; ++q) {
      const float4 f = *reinterpret_cast<const float4 *>(xs + pad(base + 4 * q));
      v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
      for (int i = 0; i < E; ++i)
        if ((i & h) == 0) {
          const float x = v[i], y = v[i + h];
          v[i] = x + y;
          v[i + h] = x - y;
        }
    const float f = sign_rows[r] * scale;
    if constexpr (E >= 16) {
      // stage 3: back through shared memory; thread (lane, warp) takes the P
      // values a*256 + m*E + bl (m < P) for bl = its lane (mod E) and E*E/256
      // values of a, and runs the last log2(P) levels in registers
#pragma unroll
      for (int q = 0; q < E / 4; ++q)
        *reinterpret_cast<float4 *>(xs + pad(base + 4 * q)) =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      __syncthreads();
      constexpr int NA = E * E / 256;                     // values of a per thread
      const int lane = t & 31, w = t >> 5;
      const int bl = lane & (E - 1);
#pragma unroll
      for (int k = 0; k < NA; ++k) {
        const int a = (E == 32) ? (w * NA + k) : (2 * w + (lane >> 4));
        float u[P];
#pragma unroll
        for (int mm = 0; mm < P; ++mm) u[mm] = xs[pad(a * 256 + mm * E + bl)];
#pragma unroll
        for (int h = 1; h < P; h <<= 1)
#pragma unroll
          for (int i = 0; i < P; ++i)
            if ((i & h) == 0) {
              const float x = u[i], y = u[i + h];
              u[i] = x + y;
              u[i + h] = x - y;
            }
        float *dst = out + (int64_t)r * C + a * 256 + bl;
#pragma unroll
        for (int mm = 0; mm < P; ++mm) dst[mm * E] = u[mm] * f;
      }
    } else {
#pragma unroll
      for (int d = 1; d < P; d <<= 1) {
        const bool upper = (m & d) != 0;
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const float o = __shfl_xor_sync(0xffffffffu, v[i], d);
          v[i] = upper ? o - v[i] : v[i] + o;
        }
      }
      float4 *dst = reinterpret_cast<float4 *>(out + (int64_t)r * C + base);
#pragma unroll
      for (int q = 0; q < E / 4; ++q)
        dst[q] = make_float4(v[4 * q] * f, v[4 * q + 1] * f, v[4 * q + 2] * f, v[4 * q + 3] * f);
    }
    __syncthreads();                                      // xs is rewritten by the next row
  }
}

// Butterflies along the rows r = hi * 2^(b0+nb) + k * 2^b0 + lo, k < 2^nb.
__global__ void __launch_bounds__(256) rht_cols_kernel(float *data, int R, int C, int b0, int nb,
                                                       float scale) {
  extern __shared__ __align__(16) float tile[];  // [2^nb][32]
  const int K = 1 << nb;
  const int n_lo = 1 << b0;
  const int n_hi = R >> (b0 + nb);
  const int n_cb = C / 32;
  const int64_t n_tiles = (int64_t)n_hi * n_lo * n_cb;
  int lcb = 0;
  while ((1 << lcb) < n_cb) ++lcb;
  for (int64_t tidx = blockIdx.x; tidx < n_tiles; tidx += gridDim.x) {
    const int cb = (int)(tidx & (n_cb - 1));            // all sizes are powers of two
    const int64_t rest = tidx >> lcb;
    const int lo = (int)(rest & (n_lo - 1)), hi = (int)(rest >> b0);
    const int64_t row0 = ((int64_t)hi << (b0 + nb)) + lo;
    for (int x = threadIdx.x; x < K * 8; x += blockDim.x) {
      const int k = x >> 3, q = x & 7;
      reinterpret_cast<float4 *>(tile)[x] =
          reinterpret_cast<const float4 *>(data + (row0 + ((int64_t)k << b0)) * C + cb * 32)[q];
    }
    __syncthreads();
    int lh = 0;
    for (; lh + 2 <= nb; lh += 2) {                     // two levels per barrier
      const int h = 1 << lh;
      for (int p = threadIdx.x; p < (K / 4) * 32; p += blockDim.x) {
        const int c = p & 31, pk = p >> 5;
        const int i = ((pk >> lh) << (lh + 2)) | (pk & (h - 1));
        float *base = tile + i * 32 + c;
        const float x0 = base[0], x1 = base[h * 32], x2 = base[2 * h * 32], x3 = base[3 * h * 32];
        const float a0 = x0 + x1, a1 = x0 - x1, a2 = x2 + x3, a3 = x2 - x3;
        base[0] = a0 + a2; base[h * 32] = a1 + a3; base[2 * h * 32] = a0 - a2; base[3 * h * 32] = a1 - a3;
      }
      __syncthreads();
    }
    if (lh < nb) {
      const int h = 1 << lh;
      for (int p = threadIdx.x; p < (K / 2) * 32; p += blockDim.x) {
        const int c = p & 31, pk = p >> 5;
        const int i = ((pk >> lh) << (lh + 1)) | (pk & (h - 1));
        const float a = tile[i * 32 + c], b = tile[(i + h) * 32 + c];
        tile[i * 32 + c] = a + b;
        tile[(i + h) * 32 + c] = a - b;
      }
      __syncthreads();
    }
    for (int x = threadIdx.x; x < K * 8; x += blockDim.x) {
      const int k = x >> 3, q = x & 7;
      float4 v = reinterpret_cast<const float4 *>(tile)[x];
      v.x *= scale; v.y *= scale; v.z *= scale; v.w *= scale;
      reinterpret_cast<float4 *>(data + (row0 + ((int64_t)k << b0)) * C + cb * 32)[q] = v;
    }
    __syncthreads();
  }
}

// Column pass over NB (6..8) row-index bits with one shared-memory round trip:
// tile = 2^NB rows r = hi 2^(b0+NB) + k 2^b0 + lo by 32 columns; lane = column
// (128-byte row segments), warp w.  Stage A: the thread holds rows k = 8j + w
// (j < E = 2^NB / 8) and runs the butterflies over the bits of j in registers;
// stage B: after a transpose through shared memory it holds, for E/8 values of
// j, the eight rows 8j + 0..7 and runs the three levels over the low bits.
template <int NB>
__global__ void __launch_bounds__(256, NB == 6 ? 8 : NB == 7 ? 4 : 2) rht_cols_reg_kernel(float *data, int R, int C, int b0,
                                                           float scale) {
  constexpr int K = 1 << NB, E = K / 8, GB = E / 8;
  static_assert(NB >= 6 && NB <= 8, "6..8 row bits per pass");
  __shared__ float tile[K * 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int n_lo = 1 << b0;
  const int n_hi = R >> (b0 + NB);
  const int n_cb = C / 32;
  int lcb = 0;
  while ((1 << lcb) < n_cb) ++lcb;
  const int64_t n_tiles = (int64_t)n_hi * n_lo * n_cb;
  for (int64_t tidx = blockIdx.x; tidx < n_tiles; tidx += gridDim.x) {
    const int cb = (int)(tidx & (n_cb - 1));
    const int64_t rest = tidx >> lcb;
    const int lo = (int)(rest & (n_lo - 1)), hi = (int)(rest >> b0);
    float *col = data + (((int64_t)hi << (b0 + NB)) + lo) * C + cb * 32 + lane;
    const int64_t rs = (int64_t)C << b0;                  // distance of rows k and k + 1
    float v[E];
#pragma unroll
    for (int j = 0; j < E; ++j) v[j] = col[(8 * j + w) * rs];
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
      for (int i = 0; i < E; ++i)
        if ((i & h) == 0) {
          const float x = v[i], y = v[i + h];
          v[i] = x + y;
          v[i + h] = x - y;
        }
#pragma unroll
    for (int j = 0; j < E; ++j) tile[(8 * j + w) * 32 + lane] = v[j];
    __syncthreads();
#pragma unroll
    for (int g = 0; g < GB; ++g) {
      const int j = w * GB + g;
      float u[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) u[x] = tile[(8 * j + x) * 32 + lane];
#pragma unroll
      for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if ((i & h) == 0) {
            const float x = u[i], y = u[i + h];
            u[i] = x + y;
            u[i + h] = x - y;
          }
#pragma unroll
      for (int x = 0; x < 8; ++x) col[(8 * j + x) * rs] = u[x] * scale;
    }
    __syncthreads();                                      // tile is rewritten by the next one
  }
}

}  // namespace tcq

using namespace tcq;
using namespace tcq_host;

static bool pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

extern "C" tcq_status_t tcq_rht(const float *W, int64_t rows, int64_t cols, const float *sign_rows,
                                const float *sign_cols, float *out, void *stream) {
  if (!pow2(rows) || !pow2(cols)) return TCQ_ERR_INVALID_ARG;
  if (rows < 32 || cols < 32 || cols > 8192 || rows > (1 << 20)) return TCQ_ERR_UNSUPPORTED;
  if (!W || !out || !sign_rows || !sign_cols || !aligned16(W) || !aligned16(out) ||
      !aligned16(sign_rows) || !aligned16(sign_cols))
    return TCQ_ERR_INVALID_ARG;
  cudaStream_t strm = (cudaStream_t)stream;
  const int R = (int)rows, C = (int)cols;
  const int sms = sm_count();
  const size_t smem_rows = sizeof(float) * (size_t)C;
  const int grid_rows = (int)std::min<int64_t>(R, (int64_t)sms * 8);
  const float rs = (float)(1.0 / std::sqrt((double)C));
  if (C >= 2048) {
    // fp32 row in registers: one launch shape per width
    if (C == 2048) rht_rows_reg_kernel<11><<<grid_rows, 256, 0, strm>>>(W, R, sign_rows, sign_cols, rs, out);
    else if (C == 4096) rht_rows_reg_kernel<12><<<grid_rows, 256, 0, strm>>>(W, R, sign_rows, sign_cols, rs, out);
    else rht_rows_reg_kernel<13><<<grid_rows, 256, 0, strm>>>(W, R, sign_rows, sign_cols, rs, out);
  } else {
    rht_rows_kernel<<<grid_rows, 256, smem_rows, strm>>>(W, R, C, sign_rows, sign_cols, rs, out);
  }
  if (launch_status() != TCQ_OK) return TCQ_ERR_CUDA;
  int bits = 0;
  while ((1 << bits) < R) ++bits;
  if (bits >= 12 && bits <= 24) {
    // column passes of 6..8 row bits each, register butterflies
    const int np = (bits + 7) / 8;
    int b0 = 0;
    for (int p = 0; p < np; ++p) {
      const int nb = (bits - b0) / (np - p);
      const int64_t tiles = (int64_t)(R >> nb) * (C / 32);
      const int grid = (int)std::min<int64_t>(tiles, (int64_t)sms * 8);
      const float sc = (p == np - 1) ? (float)(1.0 / std::sqrt((double)R)) : 1.0f;
      if (nb == 6) rht_cols_reg_kernel<6><<<grid, 256, 0, strm>>>(out, R, C, b0, sc);
      else if (nb == 7) rht_cols_reg_kernel<7><<<grid, 256, 0, strm>>>(out, R, C, b0, sc);
      else rht_cols_reg_kernel<8><<<grid, 256, 0, strm>>>(out, R, C, b0, sc);
      if (launch_status() != TCQ_OK) return TCQ_ERR_CUDA;
      b0 += nb;
    }
    return TCQ_OK;
  }
  const int passes = (bits + 9) / 10;
  int b0 = 0;
  for (int p = 0; p < passes; ++p) {
    const int nb = (bits - b0) / (passes - p);          // even split, <= 10 bits each
    const size_t smem = sizeof(float) * 32 * ((size_t)1 << nb);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(rht_cols_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return TCQ_ERR_CUDA;
    const int64_t tiles = (int64_t)(R >> nb) * (C / 32);
    const int grid = (int)std::min<int64_t>(tiles, (int64_t)sms * 8);
    const float sc = (p == passes - 1) ? (float)(1.0 / std::sqrt((double)R)) : 1.0f;
    rht_cols_kernel<<<grid, 256, smem, strm>>>(out, R, C, b0, nb, sc);
    if (launch_status() != TCQ_OK) return TCQ_ERR_CUDA;
    b0 += nb;
  }
  return TCQ_OK;
}
