"""Pins for the oracle's random-sign Hadamard rotation (QTIP blog, "The
trellis: a stateful codebook": QuIP#'s transform, +-1 signs and a Hadamard
transform from the left and the right, leaves the entries close to i.i.d.
Gaussian).

* H_2 = [[1, 1], [1, -1]] and H_n H_n^T = n I (so the rotation is orthonormal);
* the rotation preserves the Frobenius norm and is undone by its transpose;
* a fast Walsh-Hadamard transform written here (butterflies, an independent
  route) equals the dense definition;
* heavy-tailed weights come out near-Gaussian (kurtosis close to 3).
"""
import numpy as np
import pytest

import oracle


def test_hadamard_small_and_orthogonal():
    assert np.array_equal(oracle.hadamard(2), np.array([[1.0, 1.0], [1.0, -1.0]]))
    for n in (4, 64, 256):
        h = oracle.hadamard(n)
        assert np.all(np.abs(h) == 1)
        assert np.array_equal(h @ h.T, n * np.eye(n))


def _fwht_rows(x):
    x = np.array(x, dtype=np.float64)
    n = x.shape[1]
    h = 1
    while h < n:
        x = x.reshape(x.shape[0], -1, 2 * h)
        a, b = x[:, :, :h].copy(), x[:, :, h:].copy()
        x[:, :, :h], x[:, :, h:] = a + b, a - b
        x = x.reshape(x.shape[0], n)
        h *= 2
    return x


@pytest.mark.parametrize("R,C", [(16, 32), (64, 64), (128, 16)])
def test_rht_properties(R, C):
    rng = np.random.default_rng(R + C)
    W = rng.standard_normal((R, C))
    s1 = rng.integers(0, 2, R) * 2.0 - 1
    s2 = rng.integers(0, 2, C) * 2.0 - 1
    Y = oracle.rht(W, s1, s2)
    assert abs(np.linalg.norm(Y) - np.linalg.norm(W)) <= 1e-12 * np.linalg.norm(W)
    back = s1[:, None] * (oracle.hadamard(R) @ Y @ oracle.hadamard(C)) * s2[None, :] / np.sqrt(R * C)
    np.testing.assert_allclose(back, W, atol=1e-12)
    fast = _fwht_rows(_fwht_rows(s1[:, None] * W * s2[None, :]).T).T / np.sqrt(R * C)
    np.testing.assert_allclose(fast, Y, atol=1e-12)


def test_rht_gaussianises_heavy_tails():
    rng = np.random.default_rng(5)
    W = rng.standard_t(3, (256, 256))
    W /= W.std()
    Y = oracle.rht(W, rng.integers(0, 2, 256) * 2.0 - 1, rng.integers(0, 2, 256) * 2.0 - 1)
    kurt = lambda a: np.mean((a - a.mean()) ** 4) / np.var(a) ** 2
    assert kurt(W) > 6
    assert abs(kurt(Y) - 3.0) < 0.2


def test_closed_form_entries_match_the_kronecker_construction():
    h = oracle.hadamard(64)
    i, j = np.meshgrid(np.arange(64), np.arange(64), indexing="ij")
    assert np.array_equal(oracle.hadamard_entry(i, j), h)
    rng = np.random.default_rng(3)
    W = rng.standard_normal((64, 32))
    s1 = rng.integers(0, 2, 64) * 2.0 - 1
    s2 = rng.integers(0, 2, 32) * 2.0 - 1
    np.testing.assert_allclose(oracle.rht_entries(W, s1, s2, [0, 5, 63], [1, 31]),
                               oracle.rht(W, s1, s2)[[0, 5, 63]][:, [1, 31]], atol=1e-12)
