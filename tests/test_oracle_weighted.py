"""Pins for the curvature-weighted search (XOR-Trellis explainer, "Cliff
edges": each step's squared error is multiplied by that weight's D; the state
machine and the decoder are unchanged).

* brute force over every walk with the weighted energy sum_t D_t (c - s_t)^2;
* D = 1 everywhere is bit-identical to the unweighted search;
* a constant D = c at temperature temp is exactly the unweighted relaxation at
  temp / c (E scales by c), an identity independent of the recursions;
* the weighted VJP matches central finite differences;
* the search protects heavily weighted positions (the page's point).
"""
import numpy as np
import pytest

import oracle
import tcq_workloads as W


@pytest.mark.parametrize("L,T", [(4, 6), (6, 5), (8, 4)])
def test_weighted_viterbi_and_bcjr_match_brute_force(L, T):
    rng = np.random.default_rng(L * 7 + T)
    for _ in range(3):
        s = rng.standard_normal(T)
        D = np.exp(rng.uniform(np.log(0.1), np.log(10), T))
        bf = oracle.bruteforce(s, L, 0.3, D=D)
        st, mse, _ = oracle.viterbi_f64(s, L, D=D)
        assert abs(mse[0] * T - bf["min_energy"]) <= 1e-12 * max(1, bf["min_energy"])
        c = oracle.codebook_f64(L)
        assert abs(np.sum(D * (c[st[0].astype(np.int64)] - s) ** 2) - bf["min_energy"]) <= 1e-12
        soft, lz = oracle.bcjr_soft(s, L, 0.3, D=D)
        np.testing.assert_allclose(soft[0], bf["soft"], atol=1e-12)
        assert abs(lz[0] - bf["log_z"]) <= 1e-10 * max(1, abs(bf["log_z"]))


def test_unit_weights_are_bit_identical():
    s = W.gaussian(6, 5, seq_len=64)
    st0, m0 = oracle.viterbi_f32(s, 8)
    st1, m1 = oracle.viterbi_f32(s, 8, D=np.ones_like(s))
    assert np.array_equal(st0, st1) and np.array_equal(m0.view(np.uint32), m1.view(np.uint32))


def test_weighted_fp32_walk_cost_is_sequential_sum():
    s = W.gaussian(8, 9, seq_len=64)
    D = W.curvature(8, 9, seq_len=64)
    st, mse = oracle.viterbi_f32(s, 8, D=D)
    c = oracle.codebook_f32(8)
    for i in range(8):
        acc = np.float32(0.0)
        for t in range(64):
            d = np.float32(c[st[i, t]] - s[i, t])
            e = np.float32(np.float32(d * d) * D[i, t])
            acc = np.float32(acc + e)
        assert np.float32(acc / np.float32(64)) == mse[i]


@pytest.mark.parametrize("cst", [0.25, 4.0])
def test_constant_weight_is_a_temperature_change(cst):
    s = W.gaussian(2, 13, seq_len=48)
    soft_w, lz_w = oracle.bcjr_soft(s, 8, 0.2, D=np.full_like(s, cst))
    soft_u, lz_u = oracle.bcjr_soft(s, 8, 0.2 / cst)
    np.testing.assert_allclose(soft_w, soft_u, atol=1e-12)
    np.testing.assert_allclose(lz_w, lz_u, rtol=1e-12)


def test_weighted_vjp_matches_central_differences():
    rng = np.random.default_rng(21)
    L, T, temp = 6, 10, 0.5
    s = rng.standard_normal(T)
    v = rng.standard_normal(T)
    D = np.exp(rng.uniform(np.log(0.2), np.log(5), T))
    g, _ = oracle.bcjr_vjp(s, v, L, temp, D=D)

    def F(x):
        sf, _ = oracle.bcjr_soft(x, L, temp, D=D)
        return float(np.dot(v, sf[0]))

    fd = np.empty(T)
    for u in range(T):
        h = 1e-5 * max(1.0, abs(s[u]))
        e = np.zeros(T); e[u] = h
        fd[u] = (F(s + e) - F(s - e)) / (2 * h)
    np.testing.assert_allclose(g[0], fd, rtol=1e-5, atol=1e-7 * np.abs(fd).max())


def test_heavy_weights_are_protected():
    # every 8th position weighted 50x: the weighted search quantises those
    # positions more accurately than the plain search does
    s = W.gaussian(64, 17, seq_len=64)
    D = np.ones_like(s)
    D[:, ::8] = 50.0
    c = oracle.codebook_f64(8)
    st_w, _, _ = oracle.viterbi_f64(s, 8, D=D)
    st_u, _, _ = oracle.viterbi_f64(s, 8)
    err_w = np.mean((c[st_w[:, ::8].astype(np.int64)] - s[:, ::8]) ** 2)
    err_u = np.mean((c[st_u[:, ::8].astype(np.int64)] - s[:, ::8]) ** 2)
    assert err_w < 0.5 * err_u
