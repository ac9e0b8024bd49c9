/*
 * tcq_oracle.c -- plain, slow CPU oracle for bitshift-trellis coded quantisation.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the test-suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant generator
 * with the CUDA library; it is written from the pages' definitions, one
 * sequence at a time, with no blocking, fusion or reordering.
 *
 * Sources (web pages restated here in our own code):
 *   [QTIP-blog]  "QTIP: Trellis-Coded Quantization Puts 2-Bit LLM Weights 10%
 *                Above the Rate-Distortion Bound ..." (mohakchugh.is-a.dev),
 *                sections "The trellis: a stateful codebook",
 *                "The codebook is computed", "Reproducing Table 1".
 *   [BCJR-QAT]   "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded
 *                Weight Quantization", abstract (the BCJR relaxation).
 *
 * Conventions shared by every function below:
 *   L      state width in bits (2^L states), k bits per step, V = 1.
 *   T      sequence length (number of weights), s[0..T-1] the targets.
 *   code   codebook table, code[j] = value of state j (2^L entries).
 *   pred_a(j) = (j >> k) | (a << (L-k)),  a in [0, 2^k)     [QTIP-blog, trellis]
 *   succ_b(i) = ((i << k) | b) & (2^L - 1), b in [0, 2^k)
 *   Free start: every state may begin a walk with cost (code - s_0)^2.
 *   D      optional per-weight curvature (NULL = all ones).  [XOR-Trellis
 *          explainer, "Cliff edges": the squared error of step t is scaled by
 *          D_t; the trellis and the code stay as they are.]  The step cost
 *          becomes D_t (code - s_t)^2.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off (no fast-math), so
 * every float/double operation below is one IEEE-754 operation, correctly
 * rounded, in the order written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* 1MAD computed codebook   [QTIP-blog, "The codebook is computed"]          */
/* One 32-bit LCG step on the state, its byte sum (an Irwin-Hall variable   */
/* with n = 4), then centring by 510 and scaling by 1/147.8.                */
/* ------------------------------------------------------------------------ */
int orc_1mad_bytesum(uint32_t x)
{
    uint32_t y = 34038481u * x + 76625530u;          /* arithmetic mod 2^32 */
    return (int)(y & 255u) + (int)((y >> 8) & 255u) +
           (int)((y >> 16) & 255u) + (int)((y >> 24) & 255u);
}

double orc_1mad_f64(uint32_t x)
{
    return ((double)orc_1mad_bytesum(x) - 510.0) / 147.8;
}

/* fp32 codebook value: the fp64 value of the pages rounded once to fp32. */
float orc_1mad_f32(uint32_t x)
{
    return (float)orc_1mad_f64(x);
}

void orc_codebook_1mad_f64(int L, double *out)
{
    for (uint32_t j = 0; j < (1u << L); ++j) out[j] = orc_1mad_f64(j);
}

void orc_codebook_1mad_f32(int L, float *out)
{
    for (uint32_t j = 0; j < (1u << L); ++j) out[j] = orc_1mad_f32(j);
}

/* ------------------------------------------------------------------------ */
/* Viterbi, fp32 canonical arithmetic   [QTIP-blog, trellis section]         */
/*   cost_0(j) = (code_j - s_0)^2                                            */
/*   cost_t(j) = min_a cost_{t-1}(pred_a(j)) + (code_j - s_t)^2              */
/* Each fp32 step is d = code - s, e = d * d (then e = e * D_t when weights */
/* are given), cost = best + e, every one rounded to fp32 (no fused          */
/* multiply-add).  The argmin over a keeps the     */
/* first (lowest a) minimum, like numpy's argmin; the final argmin keeps the */
/* lowest state.  Returns the minimum total cost; states[0..T-1] the walk.   */
/*                                                                           */
/* min_margin (nullable): the smallest relative decision margin along the   */
/* returned walk, in fp32.  A decision is each step's choice among the 2^k  */
/* predecessors of the walk's state (candidates cost_{t-1}(pred_a)) and the */
/* final choice among all states (candidates cost_{T-1}); its margin is     */
/* (second - best) / max(best, 1e-30), subtraction and division each        */
/* rounded to fp32, where "second" is the smallest candidate strictly above */
/* the best (exact ties are settled by index identically at any precision). */
/* INFINITY when no decision had two distinct candidates.                   */
/* ------------------------------------------------------------------------ */
static float rel_gap_f32(float best, float second)
{
    float den = best > 1e-30f ? best : 1e-30f;
    float gap = second - best;
    return gap / den;
}

float orc_viterbi_f32(int L, int k, int T, const float *s, const float *D, const float *code,
                      uint16_t *states, float *min_margin)
{
    const int N = 1 << L, A = 1 << k;
    /* every step's cost vector is kept when margins are wanted, else two */
    const int keep = min_margin ? T : 2;
    float *all = (float *)malloc(sizeof(float) * (size_t)keep * N);
    int32_t *back = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * N);
    float *cost = all, *next = all + N;

    for (int j = 0; j < N; ++j) {
        float d = code[j] - s[0];
        float e = d * d;
        cost[j] = D ? e * D[0] : e;
    }
    for (int t = 1; t < T; ++t) {
        if (min_margin) next = all + (size_t)t * N;
        for (int j = 0; j < N; ++j) {
            float best = INFINITY;
            int bestp = -1;
            for (int a = 0; a < A; ++a) {
                int p = (j >> k) | (a << (L - k));
                if (bestp < 0 || cost[p] < best) { best = cost[p]; bestp = p; }
            }
            float d = code[j] - s[t];
            float e = d * d;
            if (D) e = e * D[t];
            next[j] = best + e;
            back[(size_t)t * N + j] = bestp;
        }
        float *tmp = cost; cost = next; next = tmp;
    }
    int st = 0;
    for (int j = 1; j < N; ++j)
        if (cost[j] < cost[st]) st = j;
    float total = cost[st];
    float margin = INFINITY;
    if (min_margin) {   /* final decision: the smallest cost strictly above the best */
        float second = INFINITY;
        for (int j = 0; j < N; ++j)
            if (cost[j] > total && cost[j] < second) second = cost[j];
        if (second < INFINITY) margin = fminf(margin, rel_gap_f32(total, second));
    }
    states[T - 1] = (uint16_t)st;
    for (int t = T - 1; t > 0; --t) {
        int bestp = back[(size_t)t * N + st];
        if (min_margin) {   /* the walk's decision at step t, over cost_{t-1} */
            const float *prev = all + (size_t)(t - 1) * N;
            float best = prev[bestp], second = INFINITY;
            for (int a = 0; a < A; ++a) {
                int p = (st >> k) | (a << (L - k));
                if (prev[p] > best && prev[p] < second) second = prev[p];
            }
            if (second < INFINITY) margin = fminf(margin, rel_gap_f32(best, second));
        }
        st = bestp;
        states[t - 1] = (uint16_t)st;
    }
    if (min_margin) *min_margin = margin;
    free(all); free(back);
    return total;
}

/* ------------------------------------------------------------------------ */
/* Viterbi in fp64, same recursion, plus the decision margin along the walk */
/* it returns.  At every decision (each step's argmin over the 2^k          */
/* predecessors of the chosen state, and the final argmin) the margin is    */
/* (second distinct value - best) / max(|best|, 1e-30), where "second       */
/* distinct" is the smallest candidate strictly above the best (exact ties  */
/* are settled by index identically at any precision).  *min_margin gets   */
/* the smallest such margin (INFINITY when no decision had two distinct     */
/* candidates).  Returns the minimum total cost.                            */
/* ------------------------------------------------------------------------ */
static double rel_gap(double best, double second)
{
    double den = fabs(best) > 1e-30 ? fabs(best) : 1e-30;
    return (second - best) / den;
}

double orc_viterbi_f64(int L, int k, int T, const double *s, const double *D, const double *code,
                       uint16_t *states, double *min_margin)
{
    const int N = 1 << L, A = 1 << k;
    double *cost = (double *)malloc(sizeof(double) * (size_t)T * N); /* all steps kept */
    int32_t *back = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * N);

    for (int j = 0; j < N; ++j) {
        double d = code[j] - s[0];
        cost[j] = (D ? D[0] : 1.0) * d * d;
    }
    for (int t = 1; t < T; ++t) {
        const double *prev = cost + (size_t)(t - 1) * N;
        double *cur = cost + (size_t)t * N;
        for (int j = 0; j < N; ++j) {
            double best = INFINITY;
            int bestp = -1;
            for (int a = 0; a < A; ++a) {
                int p = (j >> k) | (a << (L - k));
                if (bestp < 0 || prev[p] < best) { best = prev[p]; bestp = p; }
            }
            double d = code[j] - s[t];
            cur[j] = best + (D ? D[t] : 1.0) * d * d;
            back[(size_t)t * N + j] = bestp;
        }
    }
    const double *last = cost + (size_t)(T - 1) * N;
    int st = 0;
    for (int j = 1; j < N; ++j)
        if (last[j] < last[st]) st = j;
    double total = last[st];

    double margin = INFINITY;
    {   /* final decision */
        double second = INFINITY;
        for (int j = 0; j < N; ++j)
            if (last[j] > total && last[j] < second) second = last[j];
        if (second < INFINITY) margin = fmin(margin, rel_gap(total, second));
    }
    states[T - 1] = (uint16_t)st;
    for (int t = T - 1; t > 0; --t) {
        const double *prev = cost + (size_t)(t - 1) * N;
        int bestp = back[(size_t)t * N + st];
        double best = prev[bestp], second = INFINITY;
        for (int a = 0; a < A; ++a) {
            int p = (st >> k) | (a << (L - k));
            if (prev[p] > best && prev[p] < second) second = prev[p];
        }
        if (second < INFINITY) margin = fmin(margin, rel_gap(best, second));
        st = bestp;
        states[t - 1] = (uint16_t)st;
    }
    if (min_margin) *min_margin = margin;
    free(cost); free(back);
    return total;
}

/* ------------------------------------------------------------------------ */
/* BCJR forward-backward at temperature temp, fp64, natural-log domain.     */
/* [BCJR-QAT abstract]: the soft codeword is the Boltzmann expectation over */
/* trellis paths.  Reading used here: a walk x has energy                   */
/*   E(x) = sum_t (code[x_t] - s_t)^2    (the cost Viterbi minimises)       */
/* and probability exp(-E/temp) / Z, with a free start (every first state)  */
/* and a free end.  soft[t] = E_p[code[x_t]], *log_z = log Z.               */
/*   alpha_0(j) = -e_0(j)/temp,  alpha_t(j) = LSE_a alpha_{t-1}(pred_a j)   */
/*                                            - e_t(j)/temp                  */
/*   beta_{T-1}(i) = 0,          beta_t(i) = LSE_b [beta_{t+1}(succ_b i)     */
/*                                            - e_{t+1}(succ_b i)/temp]      */
/*   gamma_t(j) = exp(alpha_t(j) + beta_t(j) - log Z)                        */
/* If alpha_out/beta_out are non-NULL they receive the T x 2^L tables.      */
/* ------------------------------------------------------------------------ */
static double lse_array(const double *v, int n)
{
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) if (v[i] > m) m = v[i];
    if (m == -INFINITY) return m;
    double acc = 0.0;
    for (int i = 0; i < n; ++i) acc += exp(v[i] - m);
    return m + log(acc);
}

static double emis(const double *code, const double *s, const double *D, int t, int j)
{
    double d = code[j] - s[t];
    return (D ? D[t] : 1.0) * d * d;
}

static void bcjr_tables(int L, int k, int T, double temp, const double *s, const double *D,
                        const double *code, double *alpha, double *beta)
{
    const int N = 1 << L, A = 1 << k;
    double tmp[64];
    for (int j = 0; j < N; ++j) alpha[j] = -emis(code, s, D, 0, j) / temp;
    for (int t = 1; t < T; ++t)
        for (int j = 0; j < N; ++j) {
            for (int a = 0; a < A; ++a)
                tmp[a] = alpha[(size_t)(t - 1) * N + ((j >> k) | (a << (L - k)))];
            alpha[(size_t)t * N + j] = lse_array(tmp, A) - emis(code, s, D, t, j) / temp;
        }
    for (int i = 0; i < N; ++i) beta[(size_t)(T - 1) * N + i] = 0.0;
    for (int t = T - 2; t >= 0; --t)
        for (int i = 0; i < N; ++i) {
            for (int b = 0; b < A; ++b) {
                int nx = ((i << k) | b) & (N - 1);
                tmp[b] = beta[(size_t)(t + 1) * N + nx] - emis(code, s, D, t + 1, nx) / temp;
            }
            beta[(size_t)t * N + i] = lse_array(tmp, A);
        }
}

int orc_bcjr_f64(int L, int k, int T, double temp, const double *s, const double *D,
                 const double *code, double *soft, double *log_z, double *alpha_out,
                 double *beta_out)
{
    const int N = 1 << L;
    if (k > 6) return -1;
    double *alpha = alpha_out ? alpha_out : (double *)malloc(sizeof(double) * (size_t)T * N);
    double *beta = beta_out ? beta_out : (double *)malloc(sizeof(double) * (size_t)T * N);
    bcjr_tables(L, k, T, temp, s, D, code, alpha, beta);
    double lz = lse_array(alpha + (size_t)(T - 1) * N, N);
    for (int t = 0; t < T; ++t) {
        double acc = 0.0;
        for (int j = 0; j < N; ++j)
            acc += exp(alpha[(size_t)t * N + j] + beta[(size_t)t * N + j] - lz) * code[j];
        soft[t] = acc;
    }
    if (log_z) *log_z = lz;
    if (!alpha_out) free(alpha);
    if (!beta_out) free(beta);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Vector-Jacobian product of the soft codeword, fp64.                      */
/* grad[u] = d/ds_u sum_t v_t soft_t.  Differentiating the Boltzmann         */
/* expectation (E is a sum of squares, so dE/ds_u = -2(code[x_u] - s_u)):   */
/*   d soft_t / d s_u = (2 D_u/temp) Cov_p(code[x_t], code[x_u]),           */
/*   grad[u] = (2 D_u/temp) (E_p[F code[x_u]] - E_p[F] soft_u),             */
/*   F = sum_t v_t code[x_t].                                               */
/* E_p[F | x_u = j] is split by the Markov property into the prefix part    */
/* phi_u(j) (which includes v_u code_j) and the suffix part psi_u(j):       */
/*   phi_0(j) = v_0 code_j,                                                 */
/*   phi_t(j) = sum_a w_a phi_{t-1}(pred_a j) + v_t code_j,                 */
/*              w_a = softmax_a alpha_{t-1}(pred_a j)                       */
/*   psi_{T-1}(i) = 0,                                                      */
/*   psi_t(i) = sum_b r_b [v_{t+1} code(succ_b i) + psi_{t+1}(succ_b i)],   */
/*              r_b = softmax_b [beta_{t+1}(succ_b i) - e_{t+1}(succ_b i)/temp] */
/*   E_p[F code[x_u]] = sum_j gamma_u(j) code_j (phi_u(j) + psi_u(j)).      */
/* soft_out (nullable) receives the soft codeword as a by-product.          */
/* ------------------------------------------------------------------------ */
int orc_bcjr_vjp_f64(int L, int k, int T, double temp, const double *s, const double *D,
                     const double *code, const double *v, double *grad, double *soft_out)
{
    const int N = 1 << L, A = 1 << k;
    if (k > 6) return -1;
    double *alpha = (double *)malloc(sizeof(double) * (size_t)T * N);
    double *beta = (double *)malloc(sizeof(double) * (size_t)T * N);
    double *phi = (double *)malloc(sizeof(double) * (size_t)T * N);
    double *psi = (double *)malloc(sizeof(double) * (size_t)T * N);
    double *soft = (double *)malloc(sizeof(double) * (size_t)T);
    double tmp[64];
    bcjr_tables(L, k, T, temp, s, D, code, alpha, beta);
    double lz = lse_array(alpha + (size_t)(T - 1) * N, N);

    for (int j = 0; j < N; ++j) phi[j] = v[0] * code[j];
    for (int t = 1; t < T; ++t)
        for (int j = 0; j < N; ++j) {
            for (int a = 0; a < A; ++a)
                tmp[a] = alpha[(size_t)(t - 1) * N + ((j >> k) | (a << (L - k)))];
            double m = lse_array(tmp, A), acc = 0.0;
            for (int a = 0; a < A; ++a)
                acc += exp(tmp[a] - m) * phi[(size_t)(t - 1) * N + ((j >> k) | (a << (L - k)))];
            phi[(size_t)t * N + j] = acc + v[t] * code[j];
        }
    for (int i = 0; i < N; ++i) psi[(size_t)(T - 1) * N + i] = 0.0;
    for (int t = T - 2; t >= 0; --t)
        for (int i = 0; i < N; ++i) {
            for (int b = 0; b < A; ++b) {
                int nx = ((i << k) | b) & (N - 1);
                tmp[b] = beta[(size_t)(t + 1) * N + nx] - emis(code, s, D, t + 1, nx) / temp;
            }
            double m = lse_array(tmp, A), acc = 0.0;
            for (int b = 0; b < A; ++b) {
                int nx = ((i << k) | b) & (N - 1);
                acc += exp(tmp[b] - m) * (v[t + 1] * code[nx] + psi[(size_t)(t + 1) * N + nx]);
            }
            psi[(size_t)t * N + i] = acc;
        }
    double ef = 0.0;
    for (int t = 0; t < T; ++t) {
        double acc = 0.0;
        for (int j = 0; j < N; ++j)
            acc += exp(alpha[(size_t)t * N + j] + beta[(size_t)t * N + j] - lz) * code[j];
        soft[t] = acc;
        ef += v[t] * acc;
    }
    for (int u = 0; u < T; ++u) {
        double acc = 0.0;
        for (int j = 0; j < N; ++j) {
            double g = exp(alpha[(size_t)u * N + j] + beta[(size_t)u * N + j] - lz);
            acc += g * code[j] * (phi[(size_t)u * N + j] + psi[(size_t)u * N + j]);
        }
        grad[u] = (2.0 * (D ? D[u] : 1.0) / temp) * (acc - ef * soft[u]);
    }
    if (soft_out) memcpy(soft_out, soft, sizeof(double) * (size_t)T);
    free(alpha); free(beta); free(phi); free(psi); free(soft);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Brute force over every walk (tiny L, T only): the plain definitions.     */
/* A walk is a first state x_0 in [0, 2^L) and T-1 k-bit digits, with       */
/* x_t = ((x_{t-1} << k) | digit_t) & (2^L - 1); there are 2^(L + k(T-1))   */
/* of them.  Outputs: the minimum energy, the Boltzmann log Z at temp, the  */
/* expectations soft[t] = E[code[x_t]] and (if non-NULL) the T x T matrix   */
/* second[t*T+u] = E[code[x_t] code[x_u]].  Returns the walk count, or -1   */
/* if it would exceed 2^24.                                                 */
/* ------------------------------------------------------------------------ */
int64_t orc_bruteforce_f64(int L, int k, int T, double temp, const double *s, const double *D,
                           const double *code, double *min_energy, double *log_z,
                           double *soft, double *second)
{
    const int bits = L + k * (T - 1);
    if (bits > 24 || T < 1 || T > 64) return -1;
    const int64_t W = (int64_t)1 << bits;
    const uint32_t mask = (1u << L) - 1u;
    int xs[64];
    double emin = INFINITY;
    for (int pass = 0; pass < 2; ++pass) {
        double z = 0.0;
        if (pass == 1) {
            for (int t = 0; t < T; ++t) soft[t] = 0.0;
            if (second) for (int i = 0; i < T * T; ++i) second[i] = 0.0;
        }
        for (int64_t w = 0; w < W; ++w) {
            /* decode the walk: x_0 is the top L bits of the index, each later   */
            /* digit the next k bits (the bitstream read most-significant first) */
            uint64_t code_bits = (uint64_t)w;
            uint32_t x = (uint32_t)(code_bits >> (k * (T - 1))) & mask;
            double E = 0.0;
            for (int t = 0; t < T; ++t) {
                if (t > 0) {
                    uint32_t dgt = (uint32_t)(code_bits >> (k * (T - 1 - t))) & ((1u << k) - 1u);
                    x = ((x << k) | dgt) & mask;
                }
                xs[t] = (int)x;
                double d = code[x] - s[t];
                E += (D ? D[t] : 1.0) * d * d;
            }
            if (pass == 0) {
                if (E < emin) emin = E;
            } else {
                double p = exp(-(E - emin) / temp);
                z += p;
                for (int t = 0; t < T; ++t) {
                    soft[t] += p * code[xs[t]];
                    if (second)
                        for (int u = 0; u < T; ++u) second[t * T + u] += p * code[xs[t]] * code[xs[u]];
                }
            }
        }
        if (pass == 1) {
            for (int t = 0; t < T; ++t) soft[t] /= z;
            if (second) for (int i = 0; i < T * T; ++i) second[i] /= z;
            *log_z = log(z) - emin / temp;
        }
    }
    *min_energy = emin;
    return W;
}

/* ------------------------------------------------------------------------ */
/* Tail-biting search   [QTIP-blog, "Tail-biting is worth its complexity"]  */
/* A tail-biting walk also wraps: the trailing L-k bits of the last state  */
/* are the leading L-k bits of the first, so the stream is exactly k*T      */
/* bits.  With that shared value o fixed, the search is a Viterbi run whose */
/* first state must have top bits o and whose last state must have low bits */
/* o; the exact optimum is the best of the 2^(L-k) runs, one per o.         */
/* orc_viterbi_pinned_*: as orc_viterbi_* (same arithmetic and tie-breaks)  */
/* with those two restrictions; returns the minimum cost (INFINITY if no    */
/* walk satisfies them).                                                     */
/* ------------------------------------------------------------------------ */
float orc_viterbi_pinned_f32(int L, int k, int T, const float *s, const float *D,
                             const float *code, int o, uint16_t *states)
{
    const int N = 1 << L, A = 1 << k;
    const int low = (1 << (L - k)) - 1;
    float *cost = (float *)malloc(sizeof(float) * N);
    float *next = (float *)malloc(sizeof(float) * N);
    int32_t *back = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * N);

    for (int j = 0; j < N; ++j) {
        if ((j >> k) != o) { cost[j] = INFINITY; continue; }
        float d = code[j] - s[0];
        float e = d * d;
        cost[j] = D ? e * D[0] : e;
    }
    for (int t = 1; t < T; ++t) {
        for (int j = 0; j < N; ++j) {
            float best = INFINITY;
            int bestp = -1;
            for (int a = 0; a < A; ++a) {
                int p = (j >> k) | (a << (L - k));
                if (bestp < 0 || cost[p] < best) { best = cost[p]; bestp = p; }
            }
            float d = code[j] - s[t];
            float e = d * d;
            if (D) e = e * D[t];
            next[j] = best + e;
            back[(size_t)t * N + j] = bestp;
        }
        float *tmp = cost; cost = next; next = tmp;
    }
    int st = -1;
    for (int j = 0; j < N; ++j)
        if ((j & low) == o && (st < 0 || cost[j] < cost[st])) st = j;
    float total = cost[st];
    states[T - 1] = (uint16_t)st;
    for (int t = T - 1; t > 0; --t) {
        st = back[(size_t)t * N + st];
        states[t - 1] = (uint16_t)st;
    }
    free(cost); free(next); free(back);
    return total;
}

double orc_viterbi_pinned_f64(int L, int k, int T, const double *s, const double *D,
                              const double *code, int o, uint16_t *states)
{
    const int N = 1 << L, A = 1 << k;
    const int low = (1 << (L - k)) - 1;
    double *cost = (double *)malloc(sizeof(double) * N);
    double *next = (double *)malloc(sizeof(double) * N);
    int32_t *back = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * N);

    for (int j = 0; j < N; ++j) {
        double d = code[j] - s[0];
        cost[j] = (j >> k) == o ? (D ? D[0] : 1.0) * d * d : INFINITY;
    }
    for (int t = 1; t < T; ++t) {
        for (int j = 0; j < N; ++j) {
            double best = INFINITY;
            int bestp = -1;
            for (int a = 0; a < A; ++a) {
                int p = (j >> k) | (a << (L - k));
                if (bestp < 0 || cost[p] < best) { best = cost[p]; bestp = p; }
            }
            double d = code[j] - s[t];
            next[j] = best + (D ? D[t] : 1.0) * d * d;
            back[(size_t)t * N + j] = bestp;
        }
        double *tmp = cost; cost = next; next = tmp;
    }
    int st = -1;
    for (int j = 0; j < N; ++j)
        if ((j & low) == o && (st < 0 || cost[j] < cost[st])) st = j;
    double total = cost[st];
    states[T - 1] = (uint16_t)st;
    for (int t = T - 1; t > 0; --t) {
        st = back[(size_t)t * N + st];
        states[t - 1] = (uint16_t)st;
    }
    free(cost); free(next); free(back);
    return total;
}

/* Brute force over tail-biting walks only (tiny L, T): minimum energy. */
double orc_bruteforce_tailbiting_f64(int L, int k, int T, const double *s, const double *D,
                                     const double *code)
{
    const int bits = L + k * (T - 1);
    if (bits > 24 || T < 1) return NAN;
    const int64_t W = (int64_t)1 << bits;
    const uint32_t mask = (1u << L) - 1u, low = (1u << (L - k)) - 1u;
    double emin = INFINITY;
    for (int64_t w = 0; w < W; ++w) {
        uint64_t cb = (uint64_t)w;
        uint32_t x = (uint32_t)(cb >> (k * (T - 1))) & mask, x0 = x;
        double E = 0.0;
        for (int t = 0; t < T; ++t) {
            if (t > 0) {
                uint32_t dgt = (uint32_t)(cb >> (k * (T - 1 - t))) & ((1u << k) - 1u);
                x = ((x << k) | dgt) & mask;
            }
            double d = code[x] - s[t];
            E += (D ? D[t] : 1.0) * d * d;
        }
        if ((x & low) == (x0 >> k) && E < emin) emin = E;
    }
    return emin;
}
