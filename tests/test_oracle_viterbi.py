"""Pins for the oracle's Viterbi (QTIP blog, "The trellis: a stateful codebook").

* brute force over every walk (2^(L + k(T-1)) of them) gives the same minimum;
* the returned walk is a bitshift walk and its cost, summed in order, is the
  returned cost bit for bit (fp32) or to rounding (fp64);
* fp32 and fp64 walks agree except at decisions closer than 1e-6 relative;
* the free-start MSE by L printed on the page, and the monotone-code MSE;
* the MSE stays above the rate-distortion bound D(R) = 2^(-2R).
"""
import json
import os

import numpy as np
import pytest
from scipy.stats import norm

import oracle
import tcq_workloads as W

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def _is_walk(states, L, k):
    st = np.asarray(states).astype(np.int64)
    low = (1 << (L - k)) - 1
    return bool(np.all((st[1:] >> k) == (st[:-1] & low)))


@pytest.mark.parametrize("L,k,T", [(4, 2, 6), (6, 2, 5), (8, 2, 4), (4, 1, 10), (6, 3, 4)])
def test_viterbi_matches_brute_force(L, k, T):
    rng = np.random.default_rng(1000 + L * 10 + T)
    for trial in range(4):
        s = rng.standard_normal(T)
        bf = oracle.bruteforce(s, L, 1.0, k=k)
        st, mse, _ = oracle.viterbi_f64(s, L, k=k)
        assert abs(mse[0] * T - bf["min_energy"]) <= 1e-12 * max(1.0, bf["min_energy"])
        assert _is_walk(st[0], L, k)
        c = oracle.codebook_f64(L)
        path_cost = np.sum((c[st[0].astype(np.int64)] - s) ** 2)
        assert abs(path_cost - bf["min_energy"]) <= 1e-12 * max(1.0, bf["min_energy"])


@pytest.mark.parametrize("L", [4, 6, 8])
def test_fp32_viterbi_walk_cost_is_sequential_sum(L):
    s = W.gaussian(16, 7, seq_len=64)
    st, mse = oracle.viterbi_f32(s, L)
    c = oracle.codebook_f32(L)
    for i in range(s.shape[0]):
        assert _is_walk(st[i], L, 2)
        acc = np.float32(0.0)
        for t in range(s.shape[1]):
            d = np.float32(c[st[i, t]] - s[i, t])
            acc = np.float32(acc + np.float32(d * d))
        assert np.float32(acc / np.float32(s.shape[1])) == mse[i]


def test_fp32_viterbi_near_brute_force_optimum():
    rng = np.random.default_rng(5)
    for _ in range(6):
        s = rng.standard_normal(5).astype(np.float32)
        bf = oracle.bruteforce(s.astype(np.float64), 6, 1.0)
        st, _ = oracle.viterbi_f32(s, 6)
        c = oracle.codebook_f64(6)
        cost = np.sum((c[st[0].astype(np.int64)] - s.astype(np.float64)) ** 2)
        assert cost <= bf["min_energy"] * (1 + 1e-5) + 1e-12


@pytest.mark.parametrize("L", [8, 12])
def test_fp32_and_fp64_walks_agree_off_near_ties(L):
    s = W.gaussian(24 if L == 8 else 6, 11)
    st32, mse32 = oracle.viterbi_f32(s, L)
    st64, mse64, margin = oracle.viterbi_f64(s, L)
    for i in range(s.shape[0]):
        if margin[i] >= 1e-6:
            assert np.array_equal(st32[i], st64[i])
        # fp32 accumulation of 256 terms stays within 256 * 2^-24 relative
        assert abs(float(mse32[i]) - mse64[i]) <= 256 * 2.0 ** -24 * mse64[i] + 1e-7


@pytest.mark.parametrize("L,n", [(8, 200), (12, 40), (16, 12)])
def test_free_start_mse_matches_page(L, n):
    g = GOLD["free_start_mse_by_L"]
    s = W.gaussian(n, 2024 + L)
    _, mse = oracle.viterbi_f32(s, L)
    m = float(np.mean(mse))
    # page: +-0.002 run to run; the sample mean over n sequences adds
    # 3 * sd/sqrt(n) of sampling noise (per-sequence sd measured here).
    tol = g["run_to_run"] + 3 * float(np.std(mse)) / np.sqrt(n)
    assert abs(m - g[f"L{L}"]) <= tol, (m, g[f"L{L}"], tol)
    assert m > GOLD["rate_distortion_bound_2bpw"]["value"]


@pytest.mark.parametrize("L,n", [(8, 64), (12, 16)])
def test_monotone_code_loses_to_scalar_rounding(L, n):
    # Gaussian quantile of (j + 1/2) / 2^L: a codebook monotone in the state
    g = GOLD["monotone_code_mse_by_L"]
    code = norm.ppf((np.arange(1 << L) + 0.5) / (1 << L)).astype(np.float32)
    s = W.gaussian(n, 99)
    _, mse = oracle.viterbi_f32(s, L, code=code)
    m = float(np.mean(mse))
    assert abs(m - g[f"L{L}"]) <= 0.004 + 3 * float(np.std(mse)) / np.sqrt(n), m
    assert m > 0.118    # worse than the 4-level Lloyd-Max scalar quantiser on the page


# ---------------------------------------------------------------- tie-break rule
# The page's Viterbi sketch (QTIP blog, "The trellis: a stateful codebook")
# takes numpy's argmin, which keeps the FIRST minimum: at every step the
# lowest predecessor digit a -- the candidates (j >> k) | (a << (L - k)) differ
# only in their top k bits, so this is also the lowest predecessor state --
# and, at the end, the lowest state.  Among all minimum-energy walks the
# returned one is therefore the smallest when walks are compared state by
# state from the LAST step backwards.  The pins below check that rule by
# enumerating every walk on codebooks with repeated values, where exact cost
# ties are everywhere; a `<=` in place of `<` in any argmin of the oracle
# returns a different walk.

def _walks(L, k, T):
    """Every walk [2^(L + k(T-1)), T] of the bitshift trellis (free start)."""
    mask = (1 << L) - 1
    x0 = np.arange(1 << L, dtype=np.int64)
    walks = x0[:, None]
    for _ in range(1, T):
        nxt = ((walks[:, -1:] << k) | np.arange(1 << k, dtype=np.int64)[None, :]) & mask
        walks = np.concatenate([np.repeat(walks, 1 << k, axis=0), nxt.reshape(-1, 1)], axis=1)
    return walks


def _energies(walks, s, code, f32):
    """Energy of each walk summed left to right, each operation rounded in the
    given precision (the order the recursion adds the step costs in)."""
    dt = np.float32 if f32 else np.float64
    c = np.asarray(code, dtype=dt)[walks]
    acc = np.zeros(walks.shape[0], dtype=dt)
    for t in range(walks.shape[1]):
        d = (c[:, t] - dt(s[t])).astype(dt)
        acc = (acc + (d * d).astype(dt)).astype(dt)
    return acc


def _lowest_min_walk(walks, energies):
    best = walks[energies == energies.min()]
    order = np.lexsort(best.T)           # last column is the primary key
    return best[order[0]]


def test_all_ties_give_the_lowest_index_walk_by_hand():
    # all-zero codebook: every candidate of every decision ties.  Lowest digit
    # at each step and lowest final state give the all-zero walk; a `<=` slip
    # in the step argmin gives predecessor 12 (digit 3), in the final argmin
    # state 15.
    L, T = 4, 4
    s = np.array([[0.3, -0.2, 1.5, 0.0]], dtype=np.float32)
    zero = np.zeros(1 << L)
    st32, _ = oracle.viterbi_f32(s, L, code=zero.astype(np.float32))
    st64, _, _ = oracle.viterbi_f64(s, L, code=zero)
    assert st32[0].tolist() == [0, 0, 0, 0]
    assert st64[0].tolist() == [0, 0, 0, 0]
    # pinned to overlap o = 1 (first state's top 2 bits, last state's low 2
    # bits): step 1 has one finite candidate, digit 1 (state 4 | (j >> 2)),
    # step 2 ties four ways (digit 0), the end is the lowest state with low
    # bits 1: walk [4, 0, 1]
    s3 = s[:, :3]
    st, _ = oracle.viterbi_pinned_f32(s3, L, 1, code=zero.astype(np.float32))
    assert st[0].tolist() == [4, 0, 1]
    st, _ = oracle.viterbi_pinned_f64(s3, L, 1, code=zero)
    assert st[0].tolist() == [4, 0, 1]


@pytest.mark.parametrize("f32", [True, False])
def test_ties_on_repeated_code_values_match_enumeration(f32):
    L, k, T = 4, 2, 4
    rng = np.random.default_rng(4242 + f32)
    walks = _walks(L, k, T)
    n_multi = 0
    for trial in range(40):
        # three code values and integer targets: many walks share the minimum
        code = rng.integers(-1, 2, 1 << L).astype(np.float64)
        s = rng.integers(-1, 2, T).astype(np.float64)
        E = _energies(walks, s, code, f32)
        n_multi += int((E == E.min()).sum() > 1)
        want = _lowest_min_walk(walks, E)
        if f32:
            st, _ = oracle.viterbi_f32(s.astype(np.float32)[None], L, code=code.astype(np.float32))
        else:
            st, _, _ = oracle.viterbi_f64(s[None], L, code=code)
        assert st[0].tolist() == want.tolist(), (trial, code, s)
    assert n_multi >= 30                   # the cases really have tied optima


@pytest.mark.parametrize("f32", [True, False])
def test_pinned_ties_match_enumeration(f32):
    L, k, T = 4, 2, 4
    low = (1 << (L - k)) - 1
    rng = np.random.default_rng(4343 + f32)
    walks = _walks(L, k, T)
    for trial in range(30):
        code = rng.integers(-1, 2, 1 << L).astype(np.float64)
        s = rng.integers(-1, 2, T).astype(np.float64)
        o = int(rng.integers(0, 1 << (L - k)))
        ok = ((walks[:, 0] >> k) == o) & ((walks[:, -1] & low) == o)
        E = _energies(walks[ok], s, code, f32)
        want = _lowest_min_walk(walks[ok], E)
        if f32:
            st, _ = oracle.viterbi_pinned_f32(s.astype(np.float32)[None], L, o, code=code.astype(np.float32))
        else:
            st, _ = oracle.viterbi_pinned_f64(s[None], L, o, code=code)
        assert st[0].tolist() == want.tolist(), (trial, o, code, s)


# ---------------------------------------------------------------- decision margins
def _prefix_minima(s, code, L, k, f32):
    """P[t][p]: least energy of any walk prefix x_0..x_t ending in state p,
    summed left to right in the given precision, by enumerating every prefix
    (rounding is monotone, so the minimum of the rounded sums is what the
    recursion's rounded minimum gives)."""
    out = []
    for t in range(len(s)):
        walks = _walks(L, k, t + 1)
        E = _energies(walks, s[:t + 1], code, f32)
        P = np.full(1 << L, np.inf, dtype=np.float32 if f32 else np.float64)
        np.minimum.at(P, walks[:, -1], E)
        out.append(P)
    return out


def _margin_along(walk, P, L, k, f32):
    dt = np.float32 if f32 else np.float64

    def gap(c):
        best = c.min()
        above = c[c > best]
        if above.size == 0:
            return np.inf
        den = best if best > dt(1e-30) else dt(1e-30)
        return dt(dt(above.min() - best) / den)

    m = gap(P[-1])                                  # the final choice among all states
    for t in range(len(walk) - 1, 0, -1):           # the walk's choice at step t
        preds = (walk[t] >> k) | (np.arange(1 << k) << (L - k))
        m = min(m, gap(P[t - 1][preds]))
    return m


@pytest.mark.parametrize("f32", [True, False])
def test_decision_margin_matches_enumeration(f32):
    # QTIP blog, "The trellis: a stateful codebook": the walk is read back from
    # the argmins; the margin of each argmin along it is (second - best)/best
    L, k, T = 6, 2, 5
    rng = np.random.default_rng(77 + f32)
    code = oracle.codebook_f32(L) if f32 else oracle.codebook_f64(L)
    for trial in range(6):
        s = rng.standard_normal(T) * 1.3
        if f32:
            s = s.astype(np.float32)
            st, _, m = oracle.viterbi_f32(s[None], L, margin=True)
        else:
            st, _, m = oracle.viterbi_f64(s[None], L)
        P = _prefix_minima(s, code, L, k, f32)
        want = _margin_along(st[0].astype(np.int64), P, L, k, f32)
        assert m[0] == want, (trial, m[0], want)
        assert 0 < m[0] < np.inf


def test_decision_margin_with_ties_and_none():
    # all-zero codebook: every decision is an exact tie, so no decision has a
    # second distinct candidate and the margin is infinite
    s = np.array([[0.3, -0.2, 1.5]], dtype=np.float32)
    _, _, m = oracle.viterbi_f32(s, 4, code=np.zeros(16, np.float32), margin=True)
    assert m[0] == np.inf
    _, _, m = oracle.viterbi_f64(s, 4, code=np.zeros(16))
    assert m[0] == np.inf
    # repeated code values: ties everywhere, margins still match enumeration
    rng = np.random.default_rng(5)
    for trial in range(10):
        code = rng.integers(-1, 2, 16).astype(np.float32)
        s = rng.integers(-1, 2, 4).astype(np.float32)
        st, _, m = oracle.viterbi_f32(s[None], 4, code=code, margin=True)
        P = _prefix_minima(s, code, 4, 2, True)
        assert m[0] == _margin_along(st[0].astype(np.int64), P, 4, 2, True)


def test_fp32_margin_close_to_fp64_margin():
    # the two differ only by the rounding of the costs: each cost carries at
    # most T u relative error (u = 2^-24), so |m32 - m64| <= 2 (1 + m) T u + 2 u m
    s = W.gaussian(32, 19, seq_len=128)
    _, _, m32 = oracle.viterbi_f32(s, 8, margin=True)
    _, _, m64 = oracle.viterbi_f64(s, 8)
    u = 2.0 ** -24
    bound = 2 * (1 + m64) * 128 * u + 2 * u * m64
    assert np.all(np.abs(m32.astype(np.float64) - m64) <= bound)
