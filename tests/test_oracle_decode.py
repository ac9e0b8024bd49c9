"""Pins for the oracle's bitstream decode and pack.

The decode rule (QTIP blog, "The trellis: a stateful codebook"): reading the
stream most significant bit first, weight t is the L-bit number formed by
stream bits t*k .. t*k + L - 1.  Here it is evaluated on a string of '0'/'1'
characters, a route independent of the oracle's numpy bit arrays.  A
tail-biting stream (QTIP blog, "Tail-biting is worth its complexity") is
exactly k*T bits and its windows wrap around; the same rule on the stream with
its first L - k bits appended gives them.
"""
import numpy as np
import pytest

import oracle


def _to_int(words):
    v = 0
    for w in words:
        v = (v << 32) | int(w)
    return v


def _page_window(bits, nbits, t, L, k):
    text = format(bits, "b").zfill(nbits)          # stream bits, first bit first
    return int(text[t * k: t * k + L], 2)


@pytest.mark.parametrize("L,T", [(8, 13), (12, 40), (16, 256)])
def test_free_start_windows_match_page_formula(L, T):
    k = 2
    rng = np.random.default_rng(L + T)
    nw = oracle.stream_words(L, k, T, oracle.FREE_START)
    words = rng.integers(0, 2 ** 32, (3, nw), dtype=np.uint32)
    win = oracle.windows(words, L, k, T, oracle.FREE_START)
    nb = oracle.stream_nbits(L, k, T, oracle.FREE_START)
    for i in range(3):
        full = _to_int(words[i]) >> (32 * nw - nb)      # the nb-bit stream
        for t in range(T):
            assert win[i, t] == _page_window(full, nb, t, L, k)


@pytest.mark.parametrize("L", [8, 12, 16])
def test_tailbiting_windows_wrap(L):
    k, T = 2, 256
    rng = np.random.default_rng(L)
    words = rng.integers(0, 2 ** 32, (2, 16), dtype=np.uint32)
    win = oracle.windows(words, L, k, T, oracle.TAILBITING)
    for i in range(2):
        stream = _to_int(words[i])                       # exactly k*T = 512 bits
        ext = (stream << (L - k)) | (stream >> (k * T - (L - k)))
        nb = k * T + L - k
        for t in range(T):
            assert win[i, t] == _page_window(ext, nb, t, L, k)


def _random_walk(rng, n, T, L, k):
    st = np.empty((n, T), dtype=np.int64)
    st[:, 0] = rng.integers(0, 1 << L, n)
    for t in range(1, T):
        st[:, t] = ((st[:, t - 1] << k) | rng.integers(0, 1 << k, n)) & ((1 << L) - 1)
    return st


@pytest.mark.parametrize("L", [8, 12, 16])
def test_pack_then_decode_is_identity_free_start(L):
    rng = np.random.default_rng(3 * L)
    st = _random_walk(rng, 5, 256, L, 2)
    words = oracle.pack(st, L, oracle.FREE_START)
    assert words.shape[1] == oracle.stream_words(L, 2, 256, oracle.FREE_START)
    assert np.array_equal(oracle.windows(words, L, 2, 256, oracle.FREE_START), st)
    dec = oracle.decode(words, L, 256, oracle.FREE_START)
    assert np.array_equal(dec.view(np.uint16), oracle.codebook_f16(L)[st].view(np.uint16))


@pytest.mark.parametrize("L", [8, 16])
def test_pack_then_decode_is_identity_tailbiting(L):
    rng = np.random.default_rng(5 * L)
    words = rng.integers(0, 2 ** 32, (4, 16), dtype=np.uint32)
    st = oracle.windows(words, L, 2, 256, oracle.TAILBITING)     # a circular walk
    assert np.array_equal(oracle.pack(st, L, oracle.TAILBITING), words)


@pytest.mark.parametrize("L,k,T", [(4, 2, 3), (4, 2, 4), (6, 2, 3), (4, 1, 4)])
def test_stream_lengths_count_the_walks(L, k, T):
    # Every sequence of T states, kept when each state is its predecessor
    # shifted left by k bits with k new low bits (a walk of the bitshift
    # trellis).  Pack is one-to-one on walks and decode turns every stream into
    # a walk, so a layout of n stream bits must hold exactly 2^n walks: free
    # start, L bits for the first state and k per later step; tail-biting,
    # the walks whose last state's low L-k bits are the first state's high
    # L-k bits, exactly k*T bits.
    grid = np.stack(np.meshgrid(*[np.arange(1 << L)] * T, indexing="ij"), -1).reshape(-1, T)
    low = (1 << (L - k)) - 1
    walks = grid[np.all((grid[:, 1:] >> k) == (grid[:, :-1] & low), axis=1)]
    circ = walks[(walks[:, 0] >> k) == (walks[:, -1] & low)]
    assert len(walks) == 2 ** oracle.stream_nbits(L, k, T, oracle.FREE_START)
    assert len(circ) == 2 ** oracle.stream_nbits(L, k, T, oracle.TAILBITING) == 2 ** (k * T)
    for layout, w in ((oracle.FREE_START, walks), (oracle.TAILBITING, circ)):
        words = oracle.pack(w, L, layout, k=k)
        nb = oracle.stream_nbits(L, k, T, layout)
        pad = 32 * words.shape[1] - nb
        ints = [_to_int(r) for r in words]
        assert len(set(ints)) == len(w)                      # distinct streams
        assert all(v & ((1 << pad) - 1) == 0 for v in ints)  # only the first nb bits used
        assert np.array_equal(oracle.windows(words, L, k, T, layout), w)


def test_tile_layout():
    rng = np.random.default_rng(9)
    words = rng.integers(0, 2 ** 32, (4 * 6, 16), dtype=np.uint32)
    m = oracle.decode_tiles(words, 64, 96)
    seqs = oracle.decode(words, 16, 256)
    # sequence r*(cols/16)+c is the tile at (16r, 16c), row-major inside it
    for r in range(4):
        for c in range(6):
            tile = m[16 * r:16 * r + 16, 16 * c:16 * c + 16]
            assert np.array_equal(tile.reshape(-1).view(np.uint16),
                                  seqs[r * 6 + c].view(np.uint16))
