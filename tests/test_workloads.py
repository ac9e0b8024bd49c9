"""The seeded input recipes both sides draw from: deterministic, with the
shapes, tile order and distributions the workload table states."""
import numpy as np

import tcq_workloads as W


def test_every_workload_is_deterministic_and_shaped():
    for name, w in W.WORKLOADS.items():
        if w.kind in ("gaussian", "rht_block", "student_t"):
            a, b = W.sequences(name, n_limit=8), W.sequences(name, n_limit=8)
            assert a.dtype == np.float32 and a.shape == (8, W.SEQ_LEN)
            assert np.array_equal(a, b), name
        elif w.kind == "bitstream":
            a = W.streams(name)[:4]
            assert a.dtype == np.uint32 and np.array_equal(a, W.streams(name)[:4])


def test_tiles_to_sequences_reads_16x16_tiles_row_major():
    m = np.arange(32 * 48, dtype=np.float32).reshape(32, 48)
    seq = W.tiles_to_sequences(m)
    assert seq.shape == (2 * 3, 256)
    for r in range(2):
        for c in range(3):
            assert np.array_equal(seq[r * 3 + c], m[16 * r:16 * r + 16, 16 * c:16 * c + 16].ravel())


def test_rht_block_is_an_orthonormal_rotation_of_its_gaussian_draw():
    n, seed = 64, 5
    out = W.rht_block(seed, n).astype(np.float64)
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, n))
    s1 = rng.integers(0, 2, n) * 2 - 1
    s2 = rng.integers(0, 2, n) * 2 - 1
    # (H/sqrt n) is orthonormal and an involution: undoing the rotation gives
    # diag(s1) W diag(s2) back, and the Frobenius norm is kept
    h = W._sylvester(n) / np.sqrt(n)
    back = h @ out @ h
    assert np.allclose(back, s1[:, None] * w * s2[None, :], atol=1e-5)
    assert abs(np.linalg.norm(out) / np.linalg.norm(w) - 1) < 1e-6


def test_student_t_block_has_unit_variance_and_heavy_tails():
    x = W.student_t_block(9, 512, 2048).astype(np.float64)
    assert abs(x.var() - 1.0) < 0.03               # t(5) scaled by sqrt(3/5)
    k = ((x - x.mean()) ** 4).mean() / x.var() ** 2
    assert k > 5.0                                 # excess kurtosis 6 for t(5): tails beyond the Gaussian's 3


def test_curvature_is_log_uniform_on_its_range():
    d = W.curvature(64, 3).astype(np.float64)
    assert d.min() >= 0.1 * (1 - 1e-6) and d.max() <= 10.0 * (1 + 1e-6)
    logs = np.log10(d)
    assert abs(logs.mean()) < 0.05 and abs(logs.std() - 2 / np.sqrt(12)) < 0.03
