"""Seeded synthetic inputs for the bitshift-trellis workloads.

This module holds only input generation: random draws from numpy's PCG64
``default_rng(seed)``, the random-sign Hadamard rotation that prepares the
1024x1024 block, and the reshaping of a matrix into 256-weight sequences, one
per 16x16 tile.  It holds none of the method's arithmetic (no codebook, no
trellis search, no decode) and is the only module that both the CUDA path's
tests/benchmark and the CPU oracle's tests use.

Workloads (the pages' shapes and distributions):
  * gaussian:   n x 256 fp32 weights i.i.d. N(0, 1)          (QTIP blog, Table 1)
  * rht_block:  1024x1024 N(0,1) block after a seeded random-sign
                Walsh-Hadamard transform on both sides, cut into 16x16 tiles
                (QTIP blog, "The trellis" -- RHT from QuIP#; "What it buys end
                to end" -- one tile = one 256-long sequence)
  * student_t:  2048x8192 Student-t (nu = 5) rescaled to unit variance, tiled
  * bitstream:  uniform random 32-bit words, 16 per sequence = a tail-biting
                2-bit stream of 256 weights (QTIP blog, "Tail-biting")
  * curvature:  per-weight positive weights D, log-uniform on [0.1, 10], for the
                curvature-weighted search (XOR-Trellis explainer, "Cliff edges")
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEQ_LEN = 256


@dataclass(frozen=True)
class Workload:
    name: str
    L: int
    n_seq: int
    kind: str                      # gaussian | rht_block | student_t | bitstream
    seed: int
    temps: tuple = ()
    rows: int = 0
    cols: int = 0
    ops: tuple = field(default=())
    curv_seed: int = 0             # > 0: curvature-weighted search, D drawn from this seed
    concurrent: bool = False       # independent calls may run on separate streams at once


# The five workloads, seeds 1..5.
WORKLOADS = {
    "l8_gauss64": Workload("l8_gauss64", 8, 64, "gaussian", 1, (1.0, 0.1),
                           ops=("viterbi", "bcjr"), concurrent=True),
    "l12_gauss1024": Workload("l12_gauss1024", 12, 1024, "gaussian", 2, (0.05,),
                              ops=("viterbi", "pack_decode", "bcjr", "bcjr_grad")),
    "l16_rht1024": Workload("l16_rht1024", 16, 4096, "rht_block", 3, (), 1024, 1024,
                            ops=("viterbi",)),
    "l16_studentt_2048x8192": Workload("l16_studentt_2048x8192", 16, 65536, "student_t", 4,
                                       (1.0, 0.1, 0.01), 2048, 8192, ops=("bcjr",)),
    "l16_decode_8192sq": Workload("l16_decode_8192sq", 16, 262144, "bitstream", 5, (),
                                  8192, 8192, ops=("decode",)),
    # curvature-weighted variant of the L=12 workload (XOR-Trellis explainer,
    # "Cliff edges"); D log-uniform on [0.1, 10] from seed 6
    "l12_curv1024": Workload("l12_curv1024", 12, 1024, "gaussian", 2, (0.05,),
                             ops=("viterbi", "bcjr", "bcjr_grad"), curv_seed=6),
    # decode fused into a batch-1 GEMV: the 8192^2 stream of l16_decode_8192sq, x from seed 8
    "l16_gemv_8192sq": Workload("l16_gemv_8192sq", 16, 262144, "bitstream", 5, (), 8192, 8192,
                                ops=("gemv",)),
    # random-sign Hadamard rotation of an 8192x8192 Student-t (nu = 5) block
    "rht_t5_8192sq": Workload("rht_t5_8192sq", 16, 262144, "matrix_t5", 7, (), 8192, 8192,
                              ops=("rht",)),
    # soft codeword and gradient of the sum of soft codewords at L = 16 (QAT at
    # the 2-bit QTIP setting) on the 1024x1024 RHT block, temp 0.1
    "l16_rht1024_grad": Workload("l16_rht1024_grad", 16, 4096, "rht_block", 3, (0.1,), 1024, 1024,
                                 ops=("bcjr", "bcjr_grad")),
    # the 1024x1024 RHT block encoded tail-biting (exactly 2 bits per weight)
    "l16_rht1024_tb": Workload("l16_rht1024_tb", 16, 4096, "rht_block", 3, (), 1024, 1024,
                               ops=("viterbi_tb",)),
}


def weights(name: str, n_limit: int | None = None) -> np.ndarray | None:
    """Curvature weights [n, 256] of a weighted workload (None if unweighted)."""
    w = WORKLOADS[name]
    if not w.curv_seed:
        return None
    out = curvature(w.n_seq, w.curv_seed)
    return out if n_limit is None else np.ascontiguousarray(out[:n_limit])


def tiles_to_sequences(m: np.ndarray) -> np.ndarray:
    """[R, C] -> [(R/16)*(C/16), 256]: sequence r*(C/16)+c is the 16x16 tile
    at (16r, 16c), read row-major."""
    R, C = m.shape
    assert R % 16 == 0 and C % 16 == 0
    return np.ascontiguousarray(
        m.reshape(R // 16, 16, C // 16, 16).transpose(0, 2, 1, 3).reshape(-1, 256))


def gaussian(n_seq: int, seed: int, seq_len: int = SEQ_LEN) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.standard_normal((n_seq, seq_len)).astype(np.float32)


def _sylvester(n: int) -> np.ndarray:
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def rht_block(seed: int, n: int = 1024) -> np.ndarray:
    """H diag(sigma1) W diag(sigma2) H^T / n in fp64, cast to fp32 (H Sylvester
    Hadamard, so H/sqrt(n) is orthonormal and the result stays N(0,1))."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, n))
    s1 = rng.integers(0, 2, n) * 2 - 1
    s2 = rng.integers(0, 2, n) * 2 - 1
    h = _sylvester(n)
    out = (h * s1[None, :]) @ w @ (s2[:, None] * h.T) / n
    return out.astype(np.float32)


def student_t_block(seed: int, rows: int = 2048, cols: int = 8192, nu: float = 5.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.standard_t(nu, (rows, cols)) * np.sqrt((nu - 2.0) / nu)).astype(np.float32)


def curvature(n_seq: int, seed: int, seq_len: int = SEQ_LEN, lo: float = 0.1,
              hi: float = 10.0) -> np.ndarray:
    """Synthetic per-weight curvature D > 0, log-uniform on [lo, hi] (stands in
    for the LDL diagonal of a layer Hessian, which needs a model and data)."""
    rng = np.random.default_rng(seed)
    return np.exp(rng.uniform(np.log(lo), np.log(hi), (n_seq, seq_len))).astype(np.float32)


def bitstream(n_seq: int, seed: int, words: int = 16) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.integers(0, 2 ** 32, (n_seq, words), dtype=np.uint32)


def sequences(name: str, n_limit: int | None = None) -> np.ndarray:
    """Target sequences [n, 256] fp32 of a weight workload (optionally the
    first ``n_limit`` rows only, from the same draw)."""
    w = WORKLOADS[name]
    if w.kind == "gaussian":
        out = gaussian(w.n_seq, w.seed)
    elif w.kind == "rht_block":
        out = tiles_to_sequences(rht_block(w.seed, w.rows))
    elif w.kind == "student_t":
        out = tiles_to_sequences(student_t_block(w.seed, w.rows, w.cols))
    else:
        raise ValueError(f"{name} is a bitstream workload")
    return out if n_limit is None else np.ascontiguousarray(out[:n_limit])


def rotation_input(name: str):
    """(W [rows, cols] fp32, sign_rows, sign_cols) of a rotation workload."""
    w = WORKLOADS[name]
    assert w.kind == "matrix_t5"
    W = student_t_block(w.seed, w.rows, w.cols)
    rng = np.random.default_rng(w.seed + 100)
    s1 = (rng.integers(0, 2, w.rows) * 2 - 1).astype(np.float32)
    s2 = (rng.integers(0, 2, w.cols) * 2 - 1).astype(np.float32)
    return W, s1, s2


def gemv_vector(name: str) -> np.ndarray:
    w = WORKLOADS[name]
    return np.random.default_rng(8).standard_normal(w.cols).astype(np.float32)


def streams(name: str) -> np.ndarray:
    w = WORKLOADS[name]
    assert w.kind == "bitstream"
    return bitstream(w.n_seq, w.seed)
