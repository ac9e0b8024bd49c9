/*
 * tcq.h -- C ABI of the bitshift-trellis coded quantisation library (libtcq.so).
 *
 * The library computes, on one NVIDIA B200 (sm_100a), the data-parallel hot
 * path of trellis-coded weight quantisation on a bitshift trellis:
 *   - hard Viterbi (min-plus) encoding of many independent weight sequences,
 *   - the BCJR forward-backward relaxation at a temperature (soft codeword)
 *     and its vector-Jacobian product,
 *   - packing state walks into bitstreams and the sliding-window decode of
 *     those streams to fp16 weights.
 *
 * Sources:
 *   [QTIP]  blog post "QTIP: Trellis-Coded Quantization Puts 2-Bit LLM Weights
 *           10% Above the Rate-Distortion Bound, and a Monotone Codebook Loses
 *           to Scalar Rounding", sections "The trellis: a stateful codebook",
 *           "The codebook is computed", "Tail-biting is worth its complexity",
 *           "What it buys end to end".
 *   [BCJR]  "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight
 *           Quantization", abstract.
 *
 * Common conventions
 *   - The trellis is (L, k, V) with V = 1: 2^L states, each step appends k
 *     bits; the transitions out of state i go to j = ((i << k) | d) mod 2^L
 *     for the 2^k digits d [QTIP, trellis].  Supported: k = 2, V = 1,
 *     L in {8, 12, 16}, 1 <= seq_len <= 256.  Anything else returns
 *     TCQ_ERR_UNSUPPORTED.
 *   - The codebook is 1MAD [QTIP, codebook]: code(j) = (bytesum(34038481 j +
 *     76625530 mod 2^32) - 510) / 147.8.  Viterbi and BCJR use its fp32 value
 *     (the fp64 value rounded once to fp32); decode writes its fp16 value
 *     (round to nearest even).
 *   - Every array pointer is a DEVICE pointer owned by the caller, contiguous,
 *     row-major, 16-byte aligned.  The library never allocates, never frees
 *     and never synchronises the host in these calls: work is enqueued on the
 *     caller's stream (`stream` is a cudaStream_t passed as void*; NULL = the
 *     legacy default stream) and outputs are valid once that stream reaches
 *     the work.  Calls are re-entrant; two calls may share a workspace only if
 *     they are ordered on the GPU.
 *   - Arguments are validated on the host before anything is launched; on an
 *     error no work is enqueued and outputs are untouched.  A failed launch
 *     returns TCQ_ERR_CUDA (the CUDA error is left for the caller to query).
 *   - Input values are not checked: non-finite targets give unspecified
 *     outputs.
 */
#ifndef TCQ_H
#define TCQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TCQ_API __attribute__((visibility("default")))
#else
#define TCQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tcq_trellis {
    int32_t L;        /* state bits (8, 12 or 16) */
    int32_t k;        /* bits per step (2) */
    int32_t V;        /* weights per step (1) */
    int32_t seq_len;  /* weights per sequence, T (1..256) */
} tcq_trellis_t;

typedef enum tcq_status {
    TCQ_OK = 0,
    TCQ_ERR_INVALID_ARG = -1,   /* null pointer, bad size, misalignment, bad enum */
    TCQ_ERR_UNSUPPORTED = -2,   /* valid but not implemented (L, k, V, seq_len, layout) */
    TCQ_ERR_WORKSPACE = -3,     /* workspace pointer missing or smaller than required */
    TCQ_ERR_CUDA = -4           /* a CUDA call or kernel launch failed */
} tcq_status_t;

/* Bitstream layouts [QTIP, trellis; tail-biting].  Stream bit p of a sequence
 * sits in 32-bit word p / 32 at bit 31 - p % 32 (read most significant first);
 * weight t reads the window of bits [k t, k t + L).
 *   TCQ_TAILBITING: exactly k*T bits, the windows wrap around (needs k*T a
 *                   multiple of 32 and k*T >= L).
 *   TCQ_FREE_START: k*T + L - k bits, padded with zeros to whole words. */
enum { TCQ_TAILBITING = 0, TCQ_FREE_START = 1 };

/* Decode output layouts.
 *   TCQ_OUT_SEQ:    out[n_seq][seq_len].
 *   TCQ_OUT_TILE16: out[rows][cols] with sequence r*(cols/16)+c filling the
 *                   16x16 tile whose top-left element is (16r, 16c), row-major
 *                   inside the tile [QTIP, "What it buys end to end": each
 *                   16x16 tile is one 256-long sequence].  Needs seq_len = 256,
 *                   rows, cols multiples of 16 and rows*cols = 256*n_seq. */
enum { TCQ_OUT_SEQ = 0, TCQ_OUT_TILE16 = 1 };

/* Library version (major*10000 + minor*100 + patch). */
TCQ_API int tcq_version(void);

/* Static description of a status code. */
TCQ_API const char *tcq_status_string(tcq_status_t status);

/* Number of 32-bit words in one sequence's stream for `layout`, or 0 if the
 * trellis/layout is invalid. */
TCQ_API size_t tcq_stream_words(const tcq_trellis_t *trellis, int layout);

/* ------------------------------------------------------------------------
 * Viterbi encode [QTIP, trellis: Viterbi finds the walk of least squared
 * error].
 *   cost_0(j) = (code_j - s_0)^2,
 *   cost_t(j) = min_a cost_{t-1}((j >> k) | (a << (L-k))) + (code_j - s_t)^2,
 * free start, free end.  fp32 arithmetic with each operation rounded on its
 * own (d = code - s, e = d*d, cost = best + e; no fused multiply-add); ties go
 * to the lowest predecessor digit a, and the final argmin to the lowest state
 * (the first minimum, as the sketch's argmin takes it).
 *
 *   s          [n_seq][seq_len] fp32 targets (input).
 *   D          [n_seq][seq_len] fp32 per-weight curvature, or NULL for all
 *              ones [XOR-Trellis explainer, "Cliff edges": the squared
 *              error of step t is scaled by the curvature D_t].  The
 *              step cost becomes e = d*d, then e*D_t, each rounded on its own.
 *              D must be >= 0 and finite (other values: unspecified walks).
 *   states     [n_seq][seq_len] uint16: the chosen walk, state (L-bit window)
 *              of every weight (output).
 *   mse        [n_seq] fp32: minimum total cost / seq_len (output).
 *   min_margin [n_seq] fp32 (output, may be NULL): the smallest relative
 *              decision margin along the returned walk, so that a caller
 *              can count the sequences whose walk is decided by a near-tie.
 *              The decisions are each step's choice among the 2^k
 *              predecessors of the walk's state (candidates cost_{t-1}) and
 *              the final choice among all states (candidates cost_{T-1});
 *              a decision's margin is (second - best) / max(best, 1e-30),
 *              subtraction and division each rounded to fp32, with "second"
 *              the smallest candidate strictly above the best (exact ties are
 *              settled by the index rule and have no margin).  +inf when no
 *              decision had two distinct candidates.  Computing it re-runs
 *              the forward recursion once more (about twice the time).
 *   ws         device workspace of at least tcq_viterbi_workspace_size()
 *              bytes, 256-byte aligned; it holds the 2-bit backpointers.
 * Returns TCQ_OK, or an error as described above.
 * ------------------------------------------------------------------------ */
TCQ_API size_t tcq_viterbi_workspace_size(const tcq_trellis_t *trellis, int64_t n_seq);

TCQ_API tcq_status_t tcq_viterbi_encode(const tcq_trellis_t *trellis, const float *s,
                                        const float *D, int64_t n_seq, uint16_t *states,
                                        float *mse, float *min_margin, void *ws, size_t ws_bytes,
                                        void *stream);

/* ------------------------------------------------------------------------
 * Tail-biting Viterbi encode [QTIP, "Tail-biting is worth its complexity":
 * the walk closes on itself (the leading L-k bits of the first state are the
 * trailing L-k bits of the last one), so the stream holds exactly k*T bits;
 * the two-run search rotates the sequence by T/2, runs Viterbi, reads the
 * shared bits at the seam and re-runs with both ends pinned to them].
 *   Same arguments, arithmetic and tie-breaks as tcq_viterbi_encode; the
 *   output walk is tail-biting (pack it with TCQ_TAILBITING) and mse is its
 *   cost / seq_len.  Needs k*seq_len >= L.  Workspace: as tcq_viterbi_encode.
 *   `states` is also used as scratch between the two runs.
 * ------------------------------------------------------------------------ */
TCQ_API tcq_status_t tcq_viterbi_encode_tailbiting(const tcq_trellis_t *trellis, const float *s,
                                                   const float *D, int64_t n_seq,
                                                   uint16_t *states, float *mse, void *ws,
                                                   size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Allocation-free Viterbi encode (the pages have no counterpart: this is a
 * deployment convenience of this library).
 *
 * For callers that may not allocate device memory at call time -- a plugin
 * whose host owns all device memory and passes it only inputs and outputs, or
 * a deployment whose memory budget is fixed at start-up and that forbids
 * cudaMalloc afterwards.  Same computation and outputs as
 * tcq_viterbi_encode, but the backpointers live in a 32 MiB buffer that is
 * part of the library image on every GPU that loads it (held until the
 * process exits) instead of a caller workspace; nothing is allocated or freed.
 *
 *   Limit: n_seq * (seq_len - 1) * 2^(L-4) bytes <= 32 MiB (for seq_len 256:
 *   8,224 sequences at L = 8, 514 at L = 12, 32 at L = 16); larger requests
 *   return TCQ_ERR_WORKSPACE without launching.
 *   The first call on each device looks up the buffer's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture.
 *   All calls share the one buffer per device: calls whose work overlaps on
 *   the GPU (different streams without ordering) race and give wrong walks.
 *   The buffer keeps the last call's contents; every byte a call reads is
 *   written earlier by the same call, so nothing is cleared.
 * ------------------------------------------------------------------------ */
TCQ_API tcq_status_t tcq_viterbi_encode_noalloc(const tcq_trellis_t *trellis, const float *s,
                                                int64_t n_seq, uint16_t *states, float *mse,
                                                void *stream);

/* ------------------------------------------------------------------------
 * BCJR soft codeword [BCJR: the argmax of Viterbi replaced by forward-backward
 * sum-product at temperature temp; the soft codeword is the Boltzmann
 * expectation over trellis walks].  A walk x has energy
 *   E(x) = sum_t (code(x_t) - s_t)^2
 * and probability exp(-E/temp)/Z over all walks (free start, free end):
 *   soft[t] = E_p[code(x_t)],   log_z = log Z (natural log).
 * fp32, log domain (base 2 inside), renormalised every step.  At a step
 * whose target lies outside the code range, the emissions are taken relative
 * to the nearest code bound r: (code - r)(code - (2 s - r)) differs from
 * (code - s)^2 by a constant of the step, which cancels in every expectation
 * and is added back to log Z in fp64.
 *
 *   s        [n_seq][seq_len] fp32 (input); temp > 0 and finite.
 *   D        [n_seq][seq_len] fp32 curvature weights (>= 0) or NULL: the
 *            energy becomes sum_t D_t (code(x_t) - s_t)^2.
 *   soft     [n_seq][seq_len] fp32 (output).
 *   log_z    [n_seq] fp32 (output, may be NULL).
 *   ws       device workspace of at least tcq_bcjr_workspace_size(.., 0)
 *            bytes (per-step forward messages of the sequences in flight).
 * ------------------------------------------------------------------------ */
TCQ_API size_t tcq_bcjr_workspace_size(const tcq_trellis_t *trellis, int64_t n_seq, int with_grad);

TCQ_API tcq_status_t tcq_bcjr_soft(const tcq_trellis_t *trellis, const float *s, const float *D,
                                   int64_t n_seq, float temp, float *soft, float *log_z,
                                   void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Vector-Jacobian product of the soft codeword [BCJR: the relaxed code is a
 * smooth function of the targets]:
 *   grad_s[u] = sum_t grad_soft[t] d soft[t] / d s[u]
 *             = (2 D_u/temp) Cov_p( sum_t grad_soft[t] code(x_t), code(x_u) )
 *   (D_u = 1 when D is NULL; D as in tcq_bcjr_soft).
 *   soft       [n_seq][seq_len] the forward output of tcq_bcjr_soft for the
 *              same s and temp (input; used to centre the covariance).
 *   grad_soft  [n_seq][seq_len] fp32 (input), grad_s [n_seq][seq_len] (output).
 *   ws         at least tcq_bcjr_workspace_size(.., 1) bytes (one slot per
 *              sequence resident on the GPU; at seq_len 256 and L = 16 a slot
 *              is 32 MiB and one sequence runs per SM, about 5 GB on B200).
 * ------------------------------------------------------------------------ */
TCQ_API tcq_status_t tcq_bcjr_soft_backward(const tcq_trellis_t *trellis, const float *s,
                                            const float *D, int64_t n_seq, float temp,
                                            const float *soft, const float *grad_soft,
                                            float *grad_s, void *ws, size_t ws_bytes,
                                            void *stream);

/* ------------------------------------------------------------------------
 * Soft codeword and its vector-Jacobian product in one pass (same
 * definitions as tcq_bcjr_soft and tcq_bcjr_soft_backward).  For callers that
 * know the cotangent up front (e.g. the gradient of a fixed loss): one
 * forward-backward sweep yields soft, log Z and grad_s, where the two
 * separate calls take two sweeps.  The covariance is centred at the targets
 * clamped to the code range instead of at the soft codeword (an exact
 * identity; only rounding differs, and the clamp keeps it small for targets
 * far outside the range).
 *   grad_soft [n_seq][seq_len] (input); soft, log_z (outputs, each may be
 *   NULL); grad_s (output).  Workspace: tcq_bcjr_workspace_size(.., 1).
 * ------------------------------------------------------------------------ */
TCQ_API tcq_status_t tcq_bcjr_soft_and_grad(const tcq_trellis_t *trellis, const float *s,
                                            const float *D, int64_t n_seq, float temp,
                                            const float *grad_soft, float *soft, float *log_z,
                                            float *grad_s, void *ws, size_t ws_bytes,
                                            void *stream);

/* ------------------------------------------------------------------------
 * Pack walks into bitstreams [QTIP, trellis: state t is the L stream bits
 * that start at bit k t].  Stream bits [k t, k t + k) are the top k bits of
 * state t; a free-start stream ends with the low L-k bits of the last state.
 * For a valid walk (and, for TCQ_TAILBITING, a circular one) decode of the
 * result returns code(states).
 *   states [n_seq][seq_len] uint16 (input), bits [n_seq][tcq_stream_words()]
 *   uint32 (output).
 * ------------------------------------------------------------------------ */
TCQ_API tcq_status_t tcq_pack_states(const tcq_trellis_t *trellis, const uint16_t *states,
                             int64_t n_seq, int layout, uint32_t *bits, void *stream);

/* ------------------------------------------------------------------------
 * Sliding-window decode [QTIP, trellis: weight t reads the L-bit window at
 * stream bit k t, most significant first; every weight decodes on its own].
 *   bits  [n_seq][tcq_stream_words()] uint32 (input).
 *   out   fp16 bit patterns (uint16), layout per out_layout (output);
 *         rows/cols are used by TCQ_OUT_TILE16 only (pass 0 otherwise).
 * ------------------------------------------------------------------------ */
TCQ_API tcq_status_t tcq_decode(const tcq_trellis_t *trellis, const uint32_t *bits, int64_t n_seq,
                        int layout, int out_layout, int64_t rows, int64_t cols,
                        uint16_t *out, void *stream);

/* ------------------------------------------------------------------------
 * Decode fused into a matrix-vector product [QTIP, "What it buys end to end":
 * each 16x16 tile decodes straight into the matmul operand]:
 *   y[i] = sum_j W[i][j] x[j],  W [rows][cols] = the fp16 matrix that
 *   tcq_decode(.., TCQ_OUT_TILE16, rows, cols) produces from `bits`,
 * products and sums in fp32 (summation order unspecified).  The weights are
 * decoded in registers and never written.
 *   bits [rows/16 * cols/16][tcq_stream_words()] (input), x [cols] fp32
 *   (input), y [rows] fp32 (output; zeroed, then accumulated with atomics on
 *   `stream`).  seq_len must be 256.
 * ------------------------------------------------------------------------ */
TCQ_API tcq_status_t tcq_decode_gemv(const tcq_trellis_t *trellis, const uint32_t *bits, int layout,
                                     int64_t rows, int64_t cols, const float *x, float *y,
                                     void *stream);

/* ------------------------------------------------------------------------
 * Random-sign Hadamard rotation [QTIP, trellis section: QuIP#'s transform,
 * +-1 signs and a Hadamard transform applied from the left and the right,
 * leaves the weights close to i.i.d. Gaussian, so one fixed code serves all
 * layers]:
 *   out = (H_R / sqrt R) diag(sign_rows) W diag(sign_cols) (H_C / sqrt C)
 * with H_n the Sylvester Hadamard matrix (H_n[i][j] = (-1)^popcount(i & j)).
 *   W [rows][cols] fp32 (input), out [rows][cols] fp32 (output; may equal W),
 *   sign_rows [rows], sign_cols [cols] fp32 (+-1 expected; any values are
 *   applied as multipliers).  rows, cols powers of two, 32 <= cols <= 8192,
 *   32 <= rows <= 2^20.  fp32 butterflies; error ~ log2(rows*cols) rounding
 *   steps of the partial sums.
 * ------------------------------------------------------------------------ */
TCQ_API tcq_status_t tcq_rht(const float *W, int64_t rows, int64_t cols, const float *sign_rows,
                             const float *sign_cols, float *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TCQ_H */
