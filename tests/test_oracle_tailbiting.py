"""Pins for the tail-biting search (QTIP blog, "Tail-biting is worth its
complexity"): the walk wraps, the trailing L-k bits of the last state being the
leading L-k bits of the first; exact solving takes 2^(L-k) runs with the shared
bits fixed; Algorithm 4 takes two (rotate by T/2, free run, read the overlap at the seam, re-run with
both ends pinned).

* the pinned runs' best equals brute force over tail-biting walks only;
* Algorithm 4 never beats the exact optimum and matches it on small trellises;
* the walks are tail-biting and pack into exactly k*T bits that decode back;
* the MSE by L printed on the page (L=16: 0.0663 free -> 0.0697 tail-biting;
  L=12 Algorithm 4: 0.0733 in the paper, 0.0723 in the blog).
"""
import json
import os

import numpy as np
import pytest

import oracle
import tcq_workloads as W

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def _tail_biting(st, L, k=2):
    st = np.asarray(st).astype(np.int64)
    low = (1 << (L - k)) - 1
    walk = np.all((st[:, 1:] >> k) == (st[:, :-1] & low), axis=1)
    wrap = (st[:, 0] >> k) == (st[:, -1] & low)
    return walk & wrap


@pytest.mark.parametrize("L,T", [(4, 7), (6, 6), (8, 5)])
def test_exact_equals_brute_force_over_tail_biting_walks(L, T):
    rng = np.random.default_rng(40 + L + T)
    for _ in range(3):
        s = rng.standard_normal(T)
        st, mse = oracle.viterbi_tailbiting_exact_f64(s, L)
        assert abs(mse[0] * T - oracle.bruteforce_tailbiting(s, L)) <= 1e-12 * max(1, mse[0] * T)
        assert _tail_biting(st, L).all()


def test_algorithm4_matches_exact_at_L8():
    s = W.gaussian(40, 99)
    st, m4, _ = oracle.viterbi_tailbiting_alg4_f32(s, 8)
    _, me = oracle.viterbi_tailbiting_exact_f64(s, 8)
    assert _tail_biting(st, 8).all()
    assert np.all(m4 >= me * (1 - 1e-6))                   # never better than the optimum
    assert np.sum(np.abs(m4 - me) <= 1e-6 * me) >= 38       # and almost always equal


def test_algorithm4_near_exact_at_L12():
    s = W.gaussian(2, 77)
    _, m4, _ = oracle.viterbi_tailbiting_alg4_f32(s, 12)
    _, me = oracle.viterbi_tailbiting_exact_f64(s, 12)      # 1,024 pinned runs each
    assert np.all(m4 >= me * (1 - 1e-6))
    assert np.all(m4 <= me * 1.01)


def test_tail_biting_walks_pack_into_kT_bits_and_decode_back():
    s = W.gaussian(6, 5)
    st, _, _ = oracle.viterbi_tailbiting_alg4_f32(s, 12)
    words = oracle.pack(st, 12, oracle.TAILBITING)
    assert words.shape[1] == 16                               # 512 bits = 2 bits per weight
    assert np.array_equal(oracle.windows(words, 12, 2, 256, oracle.TAILBITING), st.astype(np.int64))


@pytest.mark.parametrize("L,n", [(12, 240), (16, 12)])
def test_tail_biting_mse_matches_page(L, n):
    g = GOLD["tail_biting_mse"]
    s = W.gaussian(n, 12345 if L == 12 else 3046)
    st, m4, _ = oracle.viterbi_tailbiting_alg4_f32(s, L)
    _, mf = oracle.viterbi_f32(s, L)
    assert _tail_biting(st, L).all()
    assert np.all(m4 >= mf)                                   # pinning never helps
    ref = g["L12_alg4_paper"] if L == 12 else g["L16_tail_biting"]
    tol = g["run_to_run"] + 3 * float(np.std(m4)) / np.sqrt(n)
    assert abs(float(np.mean(m4)) - ref) <= tol, (np.mean(m4), ref, tol)
    if L == 16:
        assert abs(float(np.mean(mf)) - g["L16_free_start"]) <= g["run_to_run"] + 3 * float(np.std(mf)) / np.sqrt(n)
