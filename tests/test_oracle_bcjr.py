"""Pins for the oracle's BCJR soft codeword and its gradient (BCJR-QAT abstract).

* brute force: the Boltzmann expectation over every walk and its log Z;
* the transfer-matrix route (the 1-D Ising chain the abstract names): log Z =
  log(1^T D_0 M D_1 M ... D_{T-1} 1), M the 0/1 bitshift adjacency, computed
  here with dense numpy matrices, independent of the oracle's recursions;
* posteriors sum to one at every step;
* temp -> infinity gives the uniform mean of the codebook; temp -> 0 gives
  the Viterbi codeword (the hard code the abstract says is recovered);
* the gradient matches central finite differences and the brute-force
  covariance (2/temp) Cov(code_t, code_u), a symmetric PSD matrix.
"""
import numpy as np
import pytest

import oracle
import tcq_workloads as W


@pytest.mark.parametrize("L,k,T", [(4, 2, 6), (6, 2, 5), (8, 2, 4), (4, 1, 9)])
@pytest.mark.parametrize("temp", [1.0, 0.1])
def test_soft_matches_brute_force(L, k, T, temp):
    rng = np.random.default_rng(L * 100 + T)
    s = rng.standard_normal(T)
    bf = oracle.bruteforce(s, L, temp, k=k)
    soft, lz = oracle.bcjr_soft(s, L, temp, k=k)
    np.testing.assert_allclose(soft[0], bf["soft"], rtol=0, atol=1e-12)
    assert abs(lz[0] - bf["log_z"]) <= 1e-10 * max(1, abs(bf["log_z"]))


def _transfer_matrix_logz(s, L, k, temp):
    N = 1 << L
    code = oracle.codebook_f64(L)
    M = np.zeros((N, N))
    for i in range(N):
        for b in range(1 << k):
            M[i, ((i << k) | b) & (N - 1)] = 1.0
    vec = np.exp(-(code - s[0]) ** 2 / temp)
    logscale = 0.0
    for t in range(1, len(s)):
        vec = (vec @ M) * np.exp(-(code - s[t]) ** 2 / temp)
        m = vec.max()
        vec /= m
        logscale += np.log(m)
    return np.log(vec.sum()) + logscale


@pytest.mark.parametrize("L,temp", [(6, 1.0), (8, 1.0), (8, 0.1)])
def test_log_z_matches_transfer_matrix(L, temp):
    s = W.gaussian(2, 31)
    _, lz = oracle.bcjr_soft(s, L, temp)
    for i in range(2):
        ref = _transfer_matrix_logz(s[i].astype(np.float64), L, 2, temp)
        assert abs(lz[i] - ref) <= 1e-9 * abs(ref)


def test_posteriors_sum_to_one_every_step():
    s = W.gaussian(1, 41, seq_len=64)
    soft, lz, tabs = oracle.bcjr_soft(s, 8, 0.1, return_tables=True)
    al, be = tabs[0]
    g = np.exp(al + be - lz[0])
    np.testing.assert_allclose(g.sum(axis=1), 1.0, atol=1e-12)
    np.testing.assert_allclose((g * oracle.codebook_f64(8)).sum(axis=1), soft[0], atol=1e-12)


def test_high_temperature_gives_codebook_mean():
    s = W.gaussian(1, 43, seq_len=32)
    soft, _ = oracle.bcjr_soft(s, 8, 1e7)
    np.testing.assert_allclose(soft[0], oracle.codebook_f64(8).mean(), atol=1e-5)


def test_low_temperature_recovers_viterbi_codeword():
    s = W.gaussian(4, 47, seq_len=64)
    st, _, margin = oracle.viterbi_f64(s, 8)
    code = oracle.codebook_f64(8)
    for i in range(4):
        if margin[i] < 1e-3:
            continue
        hard = code[st[i].astype(np.int64)]
        errs = []
        for temp in (1.0, 1e-1, 1e-2, 1e-3, 1e-4, 1e-5):
            soft, _ = oracle.bcjr_soft(s[i], 8, temp)
            errs.append(np.abs(soft[0] - hard).max())
        # shrinks with temp down to fp64 rounding (~1e-10 at temp 1e-5)
        assert all(a >= b for a, b in zip(errs[:5], errs[1:5])), errs
        assert max(errs[4:]) < 1e-6, errs


@pytest.mark.parametrize("temp", [1.0, 0.2])
def test_vjp_matches_central_differences(temp):
    rng = np.random.default_rng(7)
    L, T = 6, 12
    s = rng.standard_normal(T)
    v = rng.standard_normal(T)
    g, _ = oracle.bcjr_vjp(s, v, L, temp)

    def F(x):
        sf, _ = oracle.bcjr_soft(x, L, temp)
        return float(np.dot(v, sf[0]))

    fd = np.empty(T)
    for u in range(T):
        h = 1e-5 * max(1.0, abs(s[u]))
        e = np.zeros(T); e[u] = h
        fd[u] = (F(s + e) - F(s - e)) / (2 * h)
    np.testing.assert_allclose(g[0], fd, rtol=1e-5, atol=1e-7 * np.abs(fd).max())


@pytest.mark.parametrize("L,T,temp", [(4, 6, 1.0), (6, 5, 0.3)])
def test_jacobian_is_scaled_covariance(L, T, temp):
    rng = np.random.default_rng(L + T)
    s = rng.standard_normal(T)
    bf = oracle.bruteforce(s, L, temp)
    J = (2.0 / temp) * (bf["second"] - np.outer(bf["soft"], bf["soft"]))
    assert np.allclose(J, J.T)
    assert np.linalg.eigvalsh(J).min() > -1e-10
    assert np.all(np.diag(J) >= -1e-12)
    for t in range(T):
        v = np.zeros(T); v[t] = 1.0
        g, _ = oracle.bcjr_vjp(s, v, L, temp)
        np.testing.assert_allclose(g[0], J[t], atol=1e-10)
