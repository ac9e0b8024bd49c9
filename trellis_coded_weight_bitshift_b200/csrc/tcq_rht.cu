// Random-sign Hadamard rotation of a weight matrix.
//
// [QTIP blog, "The trellis: a stateful codebook"] before quantisation the
// weights get random signs, then a Hadamard matrix, on both sides (QuIP#'s
// rotation), which makes them approximately i.i.d. Gaussian:
//   out = (H_R / sqrt R) diag(sign_rows) W diag(sign_cols) (H_C / sqrt C),
// H_n the Sylvester Hadamard matrix.  The product is separable, so it runs as
// fast Walsh-Hadamard butterflies, (a, b) -> (a + b, a - b):
//   * row pass: one CTA per row; the signed row sits in shared memory (the
//     first two butterfly levels are done in registers on the 16-byte load),
//     log2(C) levels, then the row sign and 1/sqrt C on the store;
//   * column passes: tiles of 32 columns (128-byte row segments) by the
//     2^nb rows that differ only in one chunk of nb <= 10 row-index bits; the
//     chunks together cover log2(R) bits; in place; the last chunk scales by
//     1/sqrt R.
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

}  // namespace tcq

using namespace tcq;
using namespace tcq_host;

static bool pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

extern "C" tcq_status_t tcq_rht(const float *W, int64_t rows, int64_t cols, const float *sign_rows,
                                const float *sign_cols, float *out, void *stream) {
  if (!pow2(rows) || !pow2(cols)) return TCQ_ERR_INVALID_ARG;
  if (rows < 32 || cols < 32 || cols > 8192 || rows > (1 << 20)) return TCQ_ERR_UNSUPPORTED;
  if (!W || !out || !sign_rows || !sign_cols || !aligned16(W) || !aligned16(out) ||
      !aligned16(sign_cols))
    return TCQ_ERR_INVALID_ARG;
  cudaStream_t strm = (cudaStream_t)stream;
  const int R = (int)rows, C = (int)cols;
  const int sms = sm_count();
  const size_t smem_rows = sizeof(float) * (size_t)C;
  const int grid_rows = (int)std::min<int64_t>(R, (int64_t)sms * 8);
  rht_rows_kernel<<<grid_rows, 256, smem_rows, strm>>>(W, R, C, sign_rows, sign_cols,
                                                       (float)(1.0 / std::sqrt((double)C)), out);
  if (launch_status() != TCQ_OK) return TCQ_ERR_CUDA;
  int bits = 0;
  while ((1 << bits) < R) ++bits;
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
