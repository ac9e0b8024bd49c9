"""Plain CPU oracle for bitshift-trellis coded quantisation (TEST INFRASTRUCTURE).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and its
Python binding) never imports, links or calls it, and it never imports the
product: the two share nothing but the seeded input generators in
``tcq_workloads``.

The arithmetic lives in ``tcq_oracle.c`` (Viterbi, BCJR, the vector-Jacobian
product, brute force), compiled with gcc without fast-math; this module wraps
it with ctypes and adds the bitstream decode/pack, written with numpy bit
arrays straight from the window formula.

Sources (restated, not copied):
  * QTIP blog post, "QTIP: Trellis-Coded Quantization Puts 2-Bit LLM Weights
    10% Above the Rate-Distortion Bound ..." -- sections "The trellis: a
    stateful codebook" (bitshift trellis, predecessor set, decode window,
    Viterbi), "The codebook is computed" (1MAD), "Tail-biting is worth its
    complexity" (tail-biting stream of exactly k*T bits), "What it buys end to
    end" (each 16x16 tile is one 256-weight sequence).
  * "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight
    Quantization", abstract (soft codeword = Boltzmann expectation over walks).

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
what the pages print (908 distinct 1MAD values, the free-start MSE by L, the
monotone-code MSE), closed forms (Irwin-Hall moments, D(R)), brute force over
all walks, an independent transfer-matrix route to log Z, finite differences
and the pages' own window formula evaluated with Python integers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from functools import lru_cache

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tcq_oracle.c")
_LIB = os.path.join(_HERE, "libtcq_oracle.so")

TAILBITING = 0
FREE_START = 1


def build(force: bool = False) -> str:
    """Compile ``tcq_oracle.c`` into ``libtcq_oracle.so`` (IEEE, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


@lru_cache(maxsize=None)
def _lib():
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    lib.orc_1mad_bytesum.argtypes = [ctypes.c_uint32]
    lib.orc_1mad_bytesum.restype = I
    lib.orc_1mad_f64.argtypes = [ctypes.c_uint32]
    lib.orc_1mad_f64.restype = D
    lib.orc_1mad_f32.argtypes = [ctypes.c_uint32]
    lib.orc_1mad_f32.restype = ctypes.c_float
    lib.orc_codebook_1mad_f64.argtypes = [I, P]
    lib.orc_codebook_1mad_f32.argtypes = [I, P]
    lib.orc_viterbi_f32.argtypes = [I, I, I, P, P, P, P, P]
    lib.orc_viterbi_f32.restype = ctypes.c_float
    lib.orc_viterbi_f64.argtypes = [I, I, I, P, P, P, P, P]
    lib.orc_viterbi_f64.restype = D
    lib.orc_bcjr_f64.argtypes = [I, I, I, D, P, P, P, P, P, P, P]
    lib.orc_bcjr_f64.restype = I
    lib.orc_bcjr_vjp_f64.argtypes = [I, I, I, D, P, P, P, P, P, P]
    lib.orc_bcjr_vjp_f64.restype = I
    lib.orc_bruteforce_f64.argtypes = [I, I, I, D, P, P, P, P, P, P, P]
    lib.orc_bruteforce_f64.restype = ctypes.c_int64
    lib.orc_viterbi_pinned_f32.argtypes = [I, I, I, P, P, P, I, P]
    lib.orc_viterbi_pinned_f32.restype = ctypes.c_float
    lib.orc_viterbi_pinned_f64.argtypes = [I, I, I, P, P, P, I, P]
    lib.orc_viterbi_pinned_f64.restype = D
    lib.orc_bruteforce_tailbiting_f64.argtypes = [I, I, I, P, P, P]
    lib.orc_bruteforce_tailbiting_f64.restype = D
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _rows(D, n, T, dtype):
    """Per-row curvature weights [n, T] (or None = all ones)."""
    if D is None:
        return None
    D = np.ascontiguousarray(np.broadcast_to(np.asarray(D), (n, T)), dtype=dtype)
    return D


def _row_ptr(D, i):
    return None if D is None else _ptr(D[i])


def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:                                  # not Linux
        return os.cpu_count() or 1


def map_rows(fn, arrays, *args, threads: int | None = None, **kw):
    """Apply a row-wise routine of this module to contiguous row blocks of
    ``arrays`` (a list of [n, ...] arrays, passed positionally before
    ``args``) in a thread pool, and join each output along rows.  Keyword
    arrays with n rows (e.g. ``D``) are cut the same way.  The C routines run
    without the GIL, so the blocks run on separate cores; every row is still
    computed by the same plain routine, one at a time."""
    from concurrent.futures import ThreadPoolExecutor
    n = arrays[0].shape[0]
    threads = max(1, min(threads or host_threads(), n))
    edges = np.linspace(0, n, threads + 1).astype(int)

    def part(i):
        lo, hi = edges[i], edges[i + 1]
        kws = {key: (v[lo:hi] if isinstance(v, np.ndarray) and v.ndim >= 1 and v.shape[0] == n else v)
               for key, v in kw.items()}
        return fn(*[a[lo:hi] for a in arrays], *args, **kws)

    _lib()                                                  # build and load once, before the threads
    with ThreadPoolExecutor(threads) as ex:
        outs = list(ex.map(part, range(threads)))
    if not isinstance(outs[0], tuple):
        return np.concatenate(outs)
    return tuple(np.concatenate([o[j] for o in outs]) for j in range(len(outs[0])))


# --------------------------------------------------------------------------
# 1MAD codebook
# --------------------------------------------------------------------------
def bytesum_1mad(x: int) -> int:
    return int(_lib().orc_1mad_bytesum(int(x)))


@lru_cache(maxsize=None)
def codebook_f64(L: int) -> np.ndarray:
    out = np.empty(1 << L, dtype=np.float64)
    _lib().orc_codebook_1mad_f64(L, _ptr(out))
    out.setflags(write=False)
    return out


@lru_cache(maxsize=None)
def codebook_f32(L: int) -> np.ndarray:
    out = np.empty(1 << L, dtype=np.float32)
    _lib().orc_codebook_1mad_f32(L, _ptr(out))
    out.setflags(write=False)
    return out


def codebook_f16(L: int) -> np.ndarray:
    """fp16 value of each state: round-to-nearest-even of the fp64 1MAD value."""
    return codebook_f64(L).astype(np.float16)


# --------------------------------------------------------------------------
# Viterbi
# --------------------------------------------------------------------------
def viterbi_f32(s: np.ndarray, L: int, k: int = 2, code: np.ndarray | None = None, D=None,
                margin: bool = False):
    """fp32-canonical Viterbi on each row of ``s`` [n, T] (optional per-weight
    curvature ``D`` [n, T], step cost D_t (code - s_t)^2).

    Returns (states uint16 [n, T], mse float32 [n]) with mse = min cost / T
    computed in fp32; with ``margin=True`` also the smallest fp32 relative
    decision margin along each returned walk (float32 [n])."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    if s.ndim == 1:
        s = s[None]
    n, T = s.shape
    D = _rows(D, n, T, np.float32)
    code = codebook_f32(L) if code is None else np.ascontiguousarray(code, dtype=np.float32)
    states = np.empty((n, T), dtype=np.uint16)
    mse = np.empty(n, dtype=np.float32)
    mrg = np.empty(n, dtype=np.float32)
    lib = _lib()
    m = ctypes.c_float()
    for i in range(n):
        row = s[i]
        st = states[i]
        cost = lib.orc_viterbi_f32(L, k, T, _ptr(row), _row_ptr(D, i), _ptr(code), _ptr(st),
                                   ctypes.byref(m) if margin else None)
        mse[i] = np.float32(cost) / np.float32(T)
        mrg[i] = m.value if margin else np.nan
    return (states, mse, mrg) if margin else (states, mse)


def viterbi_f64(s: np.ndarray, L: int, k: int = 2, code: np.ndarray | None = None, D=None):
    """fp64 Viterbi; returns (states [n, T], mse float64 [n], min_margin [n])."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    if s.ndim == 1:
        s = s[None]
    n, T = s.shape
    D = _rows(D, n, T, np.float64)
    code = codebook_f64(L) if code is None else np.ascontiguousarray(code, dtype=np.float64)
    states = np.empty((n, T), dtype=np.uint16)
    mse = np.empty(n, dtype=np.float64)
    margin = np.empty(n, dtype=np.float64)
    lib = _lib()
    m = ctypes.c_double()
    for i in range(n):
        cost = lib.orc_viterbi_f64(L, k, T, _ptr(s[i]), _row_ptr(D, i), _ptr(code), _ptr(states[i]),
                                   ctypes.byref(m))
        mse[i] = cost / T
        margin[i] = m.value
    return states, mse, margin


# --------------------------------------------------------------------------
# Tail-biting search (QTIP blog, "Tail-biting is worth its complexity")
# --------------------------------------------------------------------------
def viterbi_pinned_f32(s: np.ndarray, L: int, overlap, k: int = 2, D=None,
                       code: np.ndarray | None = None):
    """fp32 Viterbi with the first state's top L-k bits and the last state's
    low L-k bits both equal to ``overlap`` (per row); returns (states, cost)."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    if s.ndim == 1:
        s = s[None]
    n, T = s.shape
    D = _rows(D, n, T, np.float32)
    overlap = np.broadcast_to(np.asarray(overlap, dtype=np.int64), (n,))
    code = codebook_f32(L) if code is None else np.ascontiguousarray(code, dtype=np.float32)
    states = np.empty((n, T), dtype=np.uint16)
    cost = np.empty(n, dtype=np.float32)
    for i in range(n):
        cost[i] = _lib().orc_viterbi_pinned_f32(L, k, T, _ptr(s[i]), _row_ptr(D, i), _ptr(code),
                                                int(overlap[i]), _ptr(states[i]))
    return states, cost


def viterbi_pinned_f64(s: np.ndarray, L: int, overlap, k: int = 2, D=None,
                       code: np.ndarray | None = None):
    """fp64 form of ``viterbi_pinned_f32``; returns (states, cost)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    if s.ndim == 1:
        s = s[None]
    n, T = s.shape
    D = _rows(D, n, T, np.float64)
    overlap = np.broadcast_to(np.asarray(overlap, dtype=np.int64), (n,))
    code = codebook_f64(L) if code is None else np.ascontiguousarray(code, dtype=np.float64)
    states = np.empty((n, T), dtype=np.uint16)
    cost = np.empty(n, dtype=np.float64)
    for i in range(n):
        cost[i] = _lib().orc_viterbi_pinned_f64(L, k, T, _ptr(s[i]), _row_ptr(D, i), _ptr(code),
                                                int(overlap[i]), _ptr(states[i]))
    return states, cost


def viterbi_tailbiting_alg4_f32(s: np.ndarray, L: int, k: int = 2, D=None):
    """The two-run tail-biting search: Viterbi on the sequence rotated by
    T/2, the overlap read off the seam (the top L-k bits of the state that
    lands on original position 0), then Viterbi on the original sequence with
    both ends pinned to it.  fp32, the same arithmetic as viterbi_f32.
    Returns (states [n, T] tail-biting walks, mse [n], overlap [n])."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    if s.ndim == 1:
        s = s[None]
    n, T = s.shape
    h = T // 2
    Dr = None if D is None else np.roll(_rows(D, n, T, np.float32), -h, axis=1)
    st_rot, _ = viterbi_f32(np.roll(s, -h, axis=1), L, k=k, D=Dr)
    overlap = st_rot[:, (T - h) % T].astype(np.int64) >> k     # rotated position of original 0
    states, cost = viterbi_pinned_f32(s, L, overlap, k=k, D=D)
    return states, (cost / np.float32(T)).astype(np.float32), overlap


def viterbi_tailbiting_exact_f64(s: np.ndarray, L: int, k: int = 2, D=None):
    """Exact tail-biting optimum: the best of the 2^(L-k) pinned runs (fp64).
    Returns (states [n, T], mse [n])."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    if s.ndim == 1:
        s = s[None]
    n, T = s.shape
    D = _rows(D, n, T, np.float64)
    code = codebook_f64(L)
    states = np.empty((n, T), dtype=np.uint16)
    mse = np.empty(n)
    buf = np.empty(T, dtype=np.uint16)
    for i in range(n):
        best = np.inf
        for o in range(1 << (L - k)):
            c = _lib().orc_viterbi_pinned_f64(L, k, T, _ptr(s[i]), _row_ptr(D, i), _ptr(code), o,
                                              _ptr(buf))
            if c < best:
                best = c
                states[i] = buf
        mse[i] = best / T
    return states, mse


def bruteforce_tailbiting(s: np.ndarray, L: int, k: int = 2, D=None) -> float:
    """Minimum energy over tail-biting walks only, by enumeration (tiny cases)."""
    s = np.ascontiguousarray(s, dtype=np.float64).ravel()
    T = s.shape[0]
    Dr = None if D is None else np.ascontiguousarray(np.broadcast_to(np.asarray(D), (T,)), dtype=np.float64)
    return float(_lib().orc_bruteforce_tailbiting_f64(L, k, T, _ptr(s), None if Dr is None else _ptr(Dr),
                                                      _ptr(codebook_f64(L))))


# --------------------------------------------------------------------------
# BCJR soft codeword and its vector-Jacobian product
# --------------------------------------------------------------------------
def bcjr_soft(s: np.ndarray, L: int, temp: float, k: int = 2, code: np.ndarray | None = None,
              return_tables: bool = False, D=None):
    """Soft codeword E_p[code(x_t)] and log Z per row of ``s`` (fp64)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    if s.ndim == 1:
        s = s[None]
    n, T = s.shape
    D = _rows(D, n, T, np.float64)
    code = codebook_f64(L) if code is None else np.ascontiguousarray(code, dtype=np.float64)
    soft = np.empty((n, T), dtype=np.float64)
    logz = np.empty(n, dtype=np.float64)
    tables = []
    lib = _lib()
    lz = ctypes.c_double()
    for i in range(n):
        if return_tables:
            al = np.empty((T, 1 << L)); be = np.empty((T, 1 << L))
            pa, pb = _ptr(al), _ptr(be)
        else:
            pa = pb = None
        rc = lib.orc_bcjr_f64(L, k, T, float(temp), _ptr(s[i]), _row_ptr(D, i), _ptr(code),
                              _ptr(soft[i]), ctypes.byref(lz), pa, pb)
        assert rc == 0
        logz[i] = lz.value
        if return_tables:
            tables.append((al, be))
    if return_tables:
        return soft, logz, tables
    return soft, logz


def bcjr_vjp(s: np.ndarray, v: np.ndarray, L: int, temp: float, k: int = 2,
             code: np.ndarray | None = None, D=None):
    """grad[u] = d/ds_u sum_t v_t soft_t per row (fp64); also returns soft."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    if s.ndim == 1:
        s = s[None]; v = v[None]
    n, T = s.shape
    D = _rows(D, n, T, np.float64)
    code = codebook_f64(L) if code is None else np.ascontiguousarray(code, dtype=np.float64)
    grad = np.empty((n, T)); soft = np.empty((n, T))
    lib = _lib()
    for i in range(n):
        rc = lib.orc_bcjr_vjp_f64(L, k, T, float(temp), _ptr(s[i]), _row_ptr(D, i), _ptr(code),
                                  _ptr(v[i]), _ptr(grad[i]), _ptr(soft[i]))
        assert rc == 0
    return grad, soft


def bruteforce(s: np.ndarray, L: int, temp: float, k: int = 2, code: np.ndarray | None = None,
               D=None):
    """Enumerate every walk of one sequence ``s`` [T] (tiny cases only).

    Returns dict(min_energy, log_z, soft [T], second [T, T], walks)."""
    s = np.ascontiguousarray(s, dtype=np.float64).ravel()
    T = s.shape[0]
    code = codebook_f64(L) if code is None else np.ascontiguousarray(code, dtype=np.float64)
    soft = np.empty(T); second = np.empty((T, T))
    emin = ctypes.c_double(); lz = ctypes.c_double()
    Dr = None if D is None else np.ascontiguousarray(np.broadcast_to(np.asarray(D), (T,)), dtype=np.float64)
    W = _lib().orc_bruteforce_f64(L, k, T, float(temp), _ptr(s), None if Dr is None else _ptr(Dr),
                                  _ptr(code), ctypes.byref(emin), ctypes.byref(lz), _ptr(soft),
                                  _ptr(second))
    if W < 0:
        raise ValueError("too many walks for brute force")
    return dict(min_energy=emin.value, log_z=lz.value, soft=soft, second=second, walks=W)


# --------------------------------------------------------------------------
# Bitstream: decode and pack (QTIP blog, "The trellis" decode window; the
# tail-biting stream of exactly k*T bits).  Stream bit p of a sequence sits
# in 32-bit word p // 32 at bit 31 - p % 32 (most significant first).
# --------------------------------------------------------------------------
def stream_nbits(L: int, k: int, T: int, layout: int) -> int:
    return k * T if layout == TAILBITING else k * T + L - k


def stream_words(L: int, k: int, T: int, layout: int) -> int:
    return (stream_nbits(L, k, T, layout) + 31) // 32


def _words_to_bits(words: np.ndarray) -> np.ndarray:
    words = np.ascontiguousarray(words, dtype=np.uint32)
    n = words.shape[0]
    by = words.astype(">u4").view(np.uint8).reshape(n, -1)
    return np.unpackbits(by, axis=1)          # bit p of the stream in column p


def _bits_to_words(bits: np.ndarray) -> np.ndarray:
    n = bits.shape[0]
    by = np.packbits(bits.astype(np.uint8), axis=1)
    return by.view(">u4").astype(np.uint32).reshape(n, -1)


def windows(words: np.ndarray, L: int, k: int, T: int, layout: int) -> np.ndarray:
    """State (L-bit window) of every weight: weight t reads stream bits
    [k t, k t + L), most significant first; the tail-biting stream wraps."""
    bits = _words_to_bits(words)
    nb = stream_nbits(L, k, T, layout)
    n = bits.shape[0]
    out = np.zeros((n, T), dtype=np.int64)
    for t in range(T):
        for i in range(L):
            p = k * t + i
            if layout == TAILBITING:
                p %= nb
            out[:, t] |= bits[:, p].astype(np.int64) << (L - 1 - i)
    return out


def decode(words: np.ndarray, L: int, T: int, layout: int = TAILBITING, k: int = 2) -> np.ndarray:
    """fp16 weights [n, T] (sequence order) decoded from packed streams."""
    w = windows(words, L, k, T, layout)
    return codebook_f16(L)[w]


def decode_tiles(words: np.ndarray, rows: int, cols: int, L: int = 16, layout: int = TAILBITING,
                 k: int = 2) -> np.ndarray:
    """Decode into a [rows, cols] fp16 matrix: sequence r*(cols/16)+c fills the
    16x16 tile whose top-left element is (16r, 16c), row-major inside the tile."""
    seqs = decode(words, L, 256, layout, k)
    nr, nc = rows // 16, cols // 16
    return seqs.reshape(nr, nc, 16, 16).transpose(0, 2, 1, 3).reshape(rows, cols)


def pack(states: np.ndarray, L: int, layout: int, k: int = 2) -> np.ndarray:
    """Pack walks [n, T] into streams.  Bits [k t, k t + k) are the top k bits
    of state t; a free-start stream ends with the remaining L - k bits of the
    last state.  For a valid walk this is the inverse of ``windows``."""
    states = np.asarray(states).astype(np.int64)
    n, T = states.shape
    nb = stream_nbits(L, k, T, layout)
    nw = stream_words(L, k, T, layout)
    bits = np.zeros((n, nw * 32), dtype=np.uint8)
    for t in range(T):
        for i in range(k):
            bits[:, k * t + i] = (states[:, t] >> (L - 1 - i)) & 1
    if layout == FREE_START:
        for i in range(k, L):
            bits[:, k * (T - 1) + i] = (states[:, T - 1] >> (L - 1 - i)) & 1
    assert nb <= nw * 32
    return _bits_to_words(bits)


# --------------------------------------------------------------------------
# Random-sign Hadamard rotation (QTIP blog, "The trellis: a stateful codebook":
# QuIP#'s transform, +-1 signs and a Hadamard transform from the left and the
# right).
# --------------------------------------------------------------------------
def hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_n (n a power of two): H_1 = [1],
    H_2m = [[H_m, H_m], [H_m, -H_m]]."""
    assert n >= 1 and n & (n - 1) == 0
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.kron(np.array([[1.0, 1.0], [1.0, -1.0]]), h)
    return h


def rht(W: np.ndarray, sign_rows: np.ndarray, sign_cols: np.ndarray) -> np.ndarray:
    """(H_R / sqrt R) diag(sign_rows) W diag(sign_cols) (H_C / sqrt C), fp64,
    by dense matrix products (the definition)."""
    W = np.asarray(W, dtype=np.float64)
    R, C = W.shape
    hr, hc = hadamard(R), hadamard(C)
    return (hr @ (np.asarray(sign_rows, np.float64)[:, None] * W * np.asarray(sign_cols, np.float64)[None, :])
            @ hc) / np.sqrt(R * C)


def hadamard_entry(i, j):
    """Closed form of the Sylvester matrix: H[i][j] = (-1)^popcount(i & j)."""
    x = np.bitwise_and(np.asarray(i, dtype=np.int64), np.asarray(j, dtype=np.int64))
    pc = np.zeros_like(x)
    while np.any(x):
        pc += x & 1
        x >>= 1
    return 1.0 - 2.0 * (pc & 1)


def rht_entries(W: np.ndarray, sign_rows, sign_cols, rows_idx, cols_idx) -> np.ndarray:
    """Selected entries of the rotation, each by its definition:
    out[i, j] = sum_{r,c} H_R[i,r] s1[r] W[r,c] s2[c] H_C[c,j] / sqrt(R C)."""
    W = np.asarray(W, dtype=np.float64)
    R, C = W.shape
    s1 = np.asarray(sign_rows, np.float64)
    s2 = np.asarray(sign_cols, np.float64)
    rr, cc = np.arange(R), np.arange(C)
    out = np.empty((len(rows_idx), len(cols_idx)))
    for b, j in enumerate(cols_idx):
        u = W @ (s2 * hadamard_entry(cc, j))                      # [R]
        for a, i in enumerate(rows_idx):
            out[a, b] = np.dot(hadamard_entry(i, rr) * s1, u)
    return out / np.sqrt(R * C)
