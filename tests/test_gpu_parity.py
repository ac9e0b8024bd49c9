"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Rules:
  * decode, pack and Viterbi states: bit-exact (integer results).  Viterbi
    runs in fp32 with every operation rounded on its own on both sides, so
    the MSE is bit-exact too; against the fp64 oracle the walks agree except
    on sequences with a decision closer than 1e-6 relative (counted, printed).
  * BCJR soft codeword: within 1e-4 absolute of the fp64 oracle.
  * VJP: within 1e-3 * max|g| of the fp64 oracle (fp32 accumulation of a
    covariance; see the design notes).
Full-size workloads run on the GPU in the launch configuration the benchmark
uses; the oracle checks every output it can afford and a seeded sample of the
rest, and cheap properties (valid walks, sequential MSE) are checked on all.
"""
import numpy as np
import pytest
import torch

import oracle
import tcq_workloads as W

pytestmark = pytest.mark.gpu

SOFT_ATOL = 1e-4
GRAD_RTOL_OF_MAX = 1e-3
NEAR_TIE = 1e-6          # relative decision margin below which two walks count as tied


@pytest.fixture(scope="module")
def tcq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import trellis_coded_weight_bitshift_b200 as m
    from trellis_coded_weight_bitshift_b200.build import build
    build()
    return m


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _is_walk(st, L):
    st = st.astype(np.int64)
    return np.all((st[:, 1:] >> 2) == (st[:, :-1] & ((1 << (L - 2)) - 1)), axis=1)


def _seq_mse_f32(s, st, L):
    """fp32 sequential sum of (code - s)^2 along each walk, / T."""
    c = oracle.codebook_f32(L)[st.astype(np.int64)]
    acc = np.zeros(s.shape[0], dtype=np.float32)
    for t in range(s.shape[1]):
        d = (c[:, t] - s[:, t]).astype(np.float32)
        acc = (acc + (d * d).astype(np.float32)).astype(np.float32)
    return (acc / np.float32(s.shape[1])).astype(np.float32)


# ---------------------------------------------------------------- decode / pack
def test_decode_tile16_full_8192_square(tcq):
    bits = W.streams("l16_decode_8192sq")
    out = tcq.decode(_dev(bits.view(np.int32)).view(torch.uint32), 16, 256, tcq.TAILBITING,
                     tcq.OUT_TILE16, 8192, 8192)
    got = out.cpu().numpy().view(np.uint16)
    ref = oracle.decode_tiles(bits, 8192, 8192).view(np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("L", [8, 12, 16])
@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("T", [256, 48, 16, 7])
def test_decode_seq_layouts(tcq, L, layout, T):
    if layout == 0 and (2 * T) % 32:
        pytest.skip("tail-biting needs k*T a multiple of 32")
    nw = oracle.stream_words(L, 2, T, layout)
    rng = np.random.default_rng(L * 1000 + T * 10 + layout)
    bits = rng.integers(0, 2 ** 32, (37, nw), dtype=np.uint32)
    if layout == 1:                                 # zero padding past the stream end
        nb = oracle.stream_nbits(L, 2, T, layout)
        pad = nw * 32 - nb
        if pad:
            bits[:, -1] &= np.uint32((0xFFFFFFFF << pad) & 0xFFFFFFFF)
    out = tcq.decode(_dev(bits.view(np.int32)).view(torch.uint32), L, T, layout, tcq.OUT_SEQ)
    ref = oracle.decode(bits, L, T, layout)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref.view(np.uint16))


def test_decode_tile16_free_start_small(tcq):
    rng = np.random.default_rng(77)
    st = np.empty((6 * 5, 256), dtype=np.int64)
    st[:, 0] = rng.integers(0, 1 << 16, st.shape[0])
    for t in range(1, 256):
        st[:, t] = ((st[:, t - 1] << 2) | rng.integers(0, 4, st.shape[0])) & 0xFFFF
    bits = oracle.pack(st, 16, oracle.FREE_START)
    out = tcq.decode(_dev(bits.view(np.int32)).view(torch.uint32), 16, 256, tcq.FREE_START,
                     tcq.OUT_TILE16, 96, 80)
    ref = oracle.decode_tiles(bits, 96, 80, layout=oracle.FREE_START)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("L", [8, 12, 16])
@pytest.mark.parametrize("layout", [0, 1])
def test_pack_matches_oracle_and_roundtrips(tcq, L, layout):
    rng = np.random.default_rng(L + 31 * layout)
    n, T = 41, 256
    if layout == 0:
        words = rng.integers(0, 2 ** 32, (n, 16), dtype=np.uint32)
        st = oracle.windows(words, L, 2, T, 0)
    else:
        st = np.empty((n, T), dtype=np.int64)
        st[:, 0] = rng.integers(0, 1 << L, n)
        for t in range(1, T):
            st[:, t] = ((st[:, t - 1] << 2) | rng.integers(0, 4, n)) & ((1 << L) - 1)
    bits = tcq.pack_states(_dev(st.astype(np.uint16).view(np.int16)).view(torch.uint16), L, layout)
    got = bits.cpu().view(torch.int32).numpy().view(np.uint32)
    assert np.array_equal(got, oracle.pack(st, L, layout))
    dec = tcq.decode(bits, L, T, layout, tcq.OUT_SEQ).cpu().numpy().view(np.uint16)
    assert np.array_equal(dec, oracle.codebook_f16(L)[st].view(np.uint16))


# ---------------------------------------------------------------- Viterbi
def _viterbi_gpu(tcq, s, L, margin=False, D=None):
    out = tcq.viterbi_encode(_dev(s), L, margin=margin, D=None if D is None else _dev(D))
    torch.cuda.synchronize()
    st = out[0].cpu().view(torch.int16).numpy().view(np.uint16)
    return (st,) + tuple(o.cpu().numpy() for o in out[1:])


def _same_f32(a, b):
    """Bit-for-bit equality of fp32 arrays (inf included)."""
    return np.array_equal(np.asarray(a, np.float32).view(np.uint32), np.asarray(b, np.float32).view(np.uint32))


def _margin_bound(m64, T):
    """|m32 - m64| bound: each fp32 cost carries at most T u relative error
    (u = 2^-24), plus the rounding of the gap and the division."""
    u = 2.0 ** -24
    return 2 * (1 + m64) * T * u + 2 * u * m64


@pytest.mark.parametrize("name", ["l8_gauss64", "l12_gauss1024"])
def test_viterbi_full_workload_bit_exact(tcq, name):
    w = W.WORKLOADS[name]
    s = W.sequences(name)
    st, mse = _viterbi_gpu(tcq, s, w.L)
    rst, rmse, rmg = oracle.map_rows(oracle.viterbi_f32, [s], w.L, margin=True)
    assert np.array_equal(st, rst)
    assert np.array_equal(mse.view(np.uint32), rmse.view(np.uint32))
    # the decision margins (second pass): same walks, margins bit for bit
    st2, mse2, mg = _viterbi_gpu(tcq, s, w.L, margin=True)
    assert np.array_equal(st2, rst) and _same_f32(mse2, rmse)
    assert _same_f32(mg, rmg)
    # against fp64 on every sequence: walks equal off near-ties (counted and
    # reported, from the GPU's margins and the fp64 oracle's), MSE within
    # 2e-5 relative (fp32 sums of 256 terms), margins within their bound
    st64, mse64, margin = oracle.map_rows(oracle.viterbi_f64, [s], w.L)
    near = margin < NEAR_TIE
    print(f"{name}: near-tie sequences (margin < {NEAR_TIE:g}): GPU {int((mg < NEAR_TIE).sum())}, "
          f"fp64 oracle {int(near.sum())} of {s.shape[0]}; smallest GPU margin {mg.min():.3g}")
    assert np.array_equal(st[~near], st64[~near])
    assert np.all(np.abs(mse - mse64) <= 2e-5 * mse64)
    ok = ~near
    assert np.all(np.abs(mg[ok].astype(np.float64) - margin[ok]) <= _margin_bound(margin[ok], s.shape[1]))


def test_viterbi_l16_rht_block(tcq):
    w = W.WORKLOADS["l16_rht1024"]
    s = W.sequences("l16_rht1024")
    st, mse = _viterbi_gpu(tcq, s, 16)
    assert st.shape == (4096, 256)
    assert np.all(_is_walk(st, 16))
    assert np.array_equal(_seq_mse_f32(s, st, 16).view(np.uint32), mse.view(np.uint32))
    st2, mse2, mg = _viterbi_gpu(tcq, s, 16, margin=True)          # every sequence's margin
    assert np.array_equal(st2, st) and _same_f32(mse2, mse)
    idx = np.random.default_rng(3).choice(4096, 62, replace=False)
    idx = np.concatenate([[0, 4095, int(np.argmin(mg))], idx])
    rst, rmse, rmg = oracle.map_rows(oracle.viterbi_f32, [s[idx]], 16, margin=True)
    assert np.array_equal(st[idx], rst)
    assert np.array_equal(mse[idx].view(np.uint32), rmse.view(np.uint32))
    assert _same_f32(mg[idx], rmg)
    # fp64 oracle on the same sample: walks equal off near-ties (counted and
    # reported), MSE within 2e-5 relative
    st64, mse64, margin = oracle.map_rows(oracle.viterbi_f64, [s[idx]], 16)
    near = margin < NEAR_TIE
    print(f"l16_rht1024: near-tie sequences (margin < {NEAR_TIE:g}): GPU {int((mg < NEAR_TIE).sum())} "
          f"of 4096 (smallest {mg.min():.3g}); fp64 oracle {int(near.sum())} of {len(idx)} sampled "
          f"(smallest {margin.min():.3g})")
    assert np.array_equal(st[idx][~near], st64[~near])
    assert np.all(np.abs(mse[idx] - mse64) <= 2e-5 * mse64)
    ok = ~near
    assert np.all(np.abs(mg[idx][ok].astype(np.float64) - margin[ok]) <= _margin_bound(margin[ok], 256))
    assert abs(float(mse.mean()) - 0.065) < 0.004       # page: free-start L=16 MSE


@pytest.mark.parametrize("L", [8, 12, 16])
@pytest.mark.parametrize("T,n", [(1, 3), (2, 5), (3, 1), (17, 9), (100, 2)])
def test_viterbi_edge_shapes(tcq, L, T, n):
    s = W.gaussian(n, 500 + T, seq_len=T) * np.float32(1.5)
    st, mse, mg = _viterbi_gpu(tcq, s, L, margin=True)
    rst, rmse, rmg = oracle.viterbi_f32(s, L, margin=True)
    assert np.array_equal(st, rst)
    assert np.array_equal(mse.view(np.uint32), rmse.view(np.uint32))
    assert _same_f32(mg, rmg)


def test_viterbi_ties_resolve_to_lowest_index(tcq):
    # all-zero targets on a codebook with repeated values: many exact ties
    s = np.zeros((9, 64), dtype=np.float32)
    s[1] = 0.25
    s[2, ::2] = -1.0
    st, mse, mg = _viterbi_gpu(tcq, s, 8, margin=True)
    rst, rmse, rmg = oracle.viterbi_f32(s, 8, margin=True)
    assert np.array_equal(st, rst)
    assert np.array_equal(mse.view(np.uint32), rmse.view(np.uint32))
    assert _same_f32(mg, rmg)             # exact ties have no margin


# ---------------------------------------------------------------- BCJR
def _bcjr_gpu(tcq, s, L, temp):
    soft, lz = tcq.bcjr_soft(_dev(s), L, temp)
    torch.cuda.synchronize()
    return soft.cpu().numpy(), lz.cpu().numpy()


@pytest.mark.parametrize("temp", [1.0, 0.1])
def test_bcjr_l8_full_workload(tcq, temp):
    s = W.sequences("l8_gauss64")
    soft, lz = _bcjr_gpu(tcq, s, 8, temp)
    rsoft, rlz = oracle.bcjr_soft(s, 8, temp)
    err = np.abs(soft - rsoft).max()
    print(f"L=8 temp={temp}: max |soft - oracle| = {err:.2e}")
    assert err <= SOFT_ATOL
    assert np.all(np.abs(lz - rlz) <= 1e-5 * np.abs(rlz) + 1e-4)


def test_bcjr_l12_workload(tcq):
    s = W.sequences("l12_gauss1024")
    soft, lz = _bcjr_gpu(tcq, s, 12, 0.05)
    idx = np.concatenate([[0, 1023], np.random.default_rng(12).choice(1024, 30, replace=False)])
    rsoft, rlz = oracle.bcjr_soft(s[idx], 12, 0.05)
    err = np.abs(soft[idx] - rsoft).max()
    print(f"L=12 temp=0.05: max |soft - oracle| = {err:.2e} over {len(idx)} sequences")
    assert err <= SOFT_ATOL
    assert np.all(np.abs(lz[idx] - rlz) <= 1e-5 * np.abs(rlz) + 1e-3)
    assert np.all(np.isfinite(soft))


def test_bcjr_l12_several_waves(tcq):
    # more sequences than one wave of the L = 12 CTAs (148 x 7 slots): each CTA
    # loops, and the last round has only a few active sequences
    n = 2100
    s = W.gaussian(n, 1212)
    v = W.gaussian(n, 1213)
    sd, vd = _dev(s), _dev(v)
    soft, lz = tcq.bcjr_soft(sd, 12, 0.1)
    soft2, lz2, g = tcq.bcjr_soft_and_grad(sd, 12, 0.1, vd)
    torch.cuda.synchronize()
    soft, soft2, g = soft.cpu().numpy(), soft2.cpu().numpy(), g.cpu().numpy()
    assert np.all(np.isfinite(soft)) and np.all(np.isfinite(g))
    assert np.abs(soft - soft2).max() <= SOFT_ATOL
    idx = np.array([0, 1035, 1036, 2071, 2072, 2099])
    rg, rsoft = oracle.bcjr_vjp(s[idx], v[idx], 12, 0.1)
    assert np.abs(soft[idx] - rsoft).max() <= SOFT_ATOL
    for i, j in enumerate(idx):
        assert np.abs(g[j] - rg[i]).max() <= GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()


@pytest.mark.parametrize("temp", [1.0, 0.1, 0.01])
def test_bcjr_l16_student_t(tcq, temp):
    # the whole 2048 x 8192 block in the benchmark's launch; the oracle checks
    # the first and last sequences, a seeded random one, and the eight with the
    # largest |s| (Student-t tails far outside the code range, where the fp32
    # emission kappa (code - s)^2 is largest and its rounding matters most)
    s = W.sequences("l16_studentt_2048x8192")
    soft, lz = _bcjr_gpu(tcq, s, 16, temp)
    assert np.all(np.isfinite(soft)) and np.all(np.isfinite(lz))
    c = oracle.codebook_f64(16)
    assert soft.min() >= c.min() - 1e-4 and soft.max() <= c.max() + 1e-4
    tails = np.argsort(-np.abs(s).max(1), kind="stable")[:8]
    idx = np.concatenate([[0, 65535, int(np.random.default_rng(int(temp * 100)).integers(1, 65535))],
                          tails])
    rsoft, rlz = oracle.map_rows(oracle.bcjr_soft, [s[idx]], 16, temp)
    err = np.abs(soft[idx] - rsoft).max(1)
    print(f"L=16 temp={temp}: max |soft - oracle| = {err[:3].max():.2e} (first, last, random); "
          f"tails (max|s| {np.abs(s[tails]).max(1).round(1).tolist()}): {err[3:].round(7).tolist()}")
    assert err.max() <= SOFT_ATOL
    assert np.all(np.abs(lz[idx] - rlz) <= 1e-5 * np.abs(rlz) + 1e-3)


@pytest.mark.parametrize("temp", [1.0, 0.01])
def test_bcjr_config4_full_properties(tcq, temp):
    # every one of the 65,536 Student-t sequences, at the temperatures the
    # workload ends on: the soft codeword is finite and inside the code range,
    # and log Z lies between the two bounds the Viterbi energy E_min gives
    # (Z holds the minimum walk, and is a sum over 2^(L + 2 (T - 1)) walks):
    #   -E_min/temp <= log Z <= -E_min/temp + (L + 2 (T - 1)) ln 2
    # with E_min = 256 x the walk's MSE, each side within log Z's 1e-5 relative
    s = W.sequences("l16_studentt_2048x8192")
    sd = _dev(s)
    soft, lz = tcq.bcjr_soft(sd, 16, temp)
    soft, lz = soft.cpu().numpy(), lz.cpu().numpy().astype(np.float64)
    # Viterbi in chunks of 8,192 sequences (8.5 GB of backpointers each)
    mse = np.concatenate([tcq.viterbi_encode(sd[i:i + 8192], 16)[1].cpu().numpy()
                          for i in range(0, sd.shape[0], 8192)])
    torch.cuda.empty_cache()
    c = oracle.codebook_f32(16)
    assert np.all(np.isfinite(soft)) and np.all(np.isfinite(lz))
    assert soft.min() >= c.min() - 1e-6 and soft.max() <= c.max() + 1e-6
    lo = -256.0 * mse.astype(np.float64) / temp
    slack = 1e-5 * np.abs(lo) + 1e-3
    assert np.all(lz >= lo - slack)
    assert np.all(lz <= lo + (16 + 2 * 255) * np.log(2.0) + slack)


@pytest.mark.parametrize("L", [8, 12, 16])
@pytest.mark.parametrize("T,n", [(1, 2), (2, 3), (5, 9), (33, 1)])
def test_bcjr_edge_shapes(tcq, L, T, n):
    s = W.gaussian(n, 900 + T, seq_len=T)
    soft, lz = _bcjr_gpu(tcq, s, L, 0.3)
    rsoft, rlz = oracle.bcjr_soft(s, L, 0.3)
    assert np.abs(soft - rsoft).max() <= SOFT_ATOL
    assert np.all(np.abs(lz - rlz) <= 1e-5 * np.abs(rlz) + 1e-4)


def _extreme_targets(T=40):
    # zeros (many exact cost ties), beyond the largest code value, far outside
    # the code range, alternating +-50, and tiny values
    rows = [np.zeros(T), np.full(T, 3.4506), np.full(T, -10.0), np.full(T, 100.0),
            np.where(np.arange(T) % 2 == 0, 50.0, -50.0),
            np.random.default_rng(77).standard_normal(T) * 1e-3]
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("L", [8, 12, 16])
def test_viterbi_extreme_targets(tcq, L):
    s = _extreme_targets()
    st, mse, mg = _viterbi_gpu(tcq, s, L, margin=True)
    rst, rmse, rmg = oracle.viterbi_f32(s, L, margin=True)
    assert np.array_equal(st, rst)
    assert np.array_equal(mse.view(np.uint32), rmse.view(np.uint32))
    assert _same_f32(mg, rmg)


@pytest.mark.parametrize("L", [8, 12, 16])
@pytest.mark.parametrize("temp", [0.1, 1.0, 1e4])
def test_bcjr_extreme_targets_and_temperatures(tcq, L, temp):
    s = _extreme_targets()
    soft, lz = _bcjr_gpu(tcq, s, L, temp)
    rsoft, rlz = oracle.bcjr_soft(s, L, temp)
    assert np.all(np.isfinite(soft)) and np.all(np.isfinite(lz))
    assert np.abs(soft - rsoft).max() <= SOFT_ATOL, np.abs(soft - rsoft).max(axis=1)
    assert np.all(np.abs(lz - rlz) <= 1e-5 * np.abs(rlz) + 1e-3)


def _beyond_range_tolerance(s, L, temp):
    # Per-row bound on the soft codeword at targets outside the code range.
    # The emission of such a step is taken relative to the nearest bound code
    # r, as (c - r)(c - (2 s - r)) = (c - s)^2 - (r - s)^2.  When the bound
    # code's state cannot repeat (L = 8: the smallest code is not on a
    # self-loop), the walks that compete alternate between the codes nearest
    # the bound, with log2 emissions up to kappa 2 |s - r| D3^2 (D3 = span of
    # the three codes nearest the bound).  Each step rounds such a value to
    # 2^-24 relative, over T steps that moves their relative weights by
    # ln2 T 2^-24 kappa 2 |s - r| D3^2, and the soft codeword by that much
    # times the codes' spread (< 1).  At L >= 12 the bound codes are dense and
    # the walks that compete stay within 1e-4.
    c = np.sort(oracle.codebook_f32(L).astype(np.float64))
    lo, hi = c[0], c[-1]
    d_lo, d_hi = c[2] - c[0], c[-1] - c[-3]
    kappa = np.log2(np.e) / temp
    T = s.shape[1]
    tol = np.full(s.shape[0], SOFT_ATOL)
    if L == 8:
        for i, row in enumerate(s.astype(np.float64)):
            ex = max(np.max(lo - row) * d_lo ** 2, np.max(row - hi) * d_hi ** 2, 0.0)
            tol[i] += np.log(2) * T * 2.0 ** -24 * kappa * 2 * ex
    return tol


@pytest.mark.parametrize("L", [8, 12, 16])
@pytest.mark.parametrize("temp", [1e-2, 1e-3])
def test_bcjr_extreme_targets_low_temperature(tcq, L, temp):
    # targets far outside the code range at low temperature: the emission of
    # such a step is taken relative to the nearest code bound, so the states
    # that compete carry small, accurately rounded emissions and exact ties
    # stay exact; log Z gets the removed constants back in fp64
    s = _extreme_targets()
    soft, lz = _bcjr_gpu(tcq, s, L, temp)
    rsoft, rlz = oracle.bcjr_soft(s, L, temp)
    assert np.all(np.isfinite(soft)) and np.all(np.isfinite(lz))
    assert np.all(np.abs(lz - rlz) <= 1e-5 * np.abs(rlz) + 1e-3)
    err = np.abs(soft - rsoft).max(axis=1)
    tol = _beyond_range_tolerance(s, L, temp)
    print(f"L={L} temp={temp:g}: max |soft - oracle| per row {err.round(8).tolist()}, "
          f"bound {tol.round(6).tolist()}")
    assert np.all(err <= tol)


def _outlier_rows(n, seed, T=64):
    # Gaussian rows with a few Student-t-sized outliers (|s| from 8 to 40), as
    # in the tails of a heavy-tailed weight block
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((n, T))
    for i in range(n):
        pos = rng.choice(T, size=3, replace=False)
        s[i, pos] = rng.choice([-1.0, 1.0], 3) * rng.uniform(8.0, 40.0, 3)
    return s.astype(np.float32)


@pytest.mark.parametrize("L", [8, 12, 16])
def test_vjp_extreme_targets(tcq, L):
    # The gradient at targets outside the code range, both entry points, on
    # rows with Student-t-sized outliers and on the constant rows of
    # _extreme_targets.  grad_u = (2/temp) Cov(F, c_u) with
    # F = sum_t v_t (c_t - m_t) is formed from fp32 sums whose terms are
    # bounded by sum_t |v_t| max|c|; a few roundings of 2^-24 each give the
    # absolute floor (2/temp) 2^-22 sum_t |v_t| max|c|, which matters where
    # the walk distribution is nearly a point mass and the exact gradient is
    # tiny.  Elsewhere the bound is 1e-3 of the row's largest entry.
    cmax = float(np.abs(oracle.codebook_f32(L)).max())
    for s in (_outlier_rows(6, 4200 + L), _extreme_targets()):
        v = W.gaussian(s.shape[0], 4100 + L, seq_len=s.shape[1])
        sd, vd = _dev(s), _dev(v)
        for temp in (0.1, 1e-2):
            soft, _ = tcq.bcjr_soft(sd, L, temp)
            g1 = tcq.bcjr_soft_backward(sd, L, temp, soft, vd)
            _, _, g2 = tcq.bcjr_soft_and_grad(sd, L, temp, vd)
            torch.cuda.synchronize()
            rg, _ = oracle.map_rows(oracle.bcjr_vjp, [s, v], L, temp)
            for g in (g1.cpu().numpy(), g2.cpu().numpy()):
                assert np.all(np.isfinite(g))
                for i in range(s.shape[0]):
                    tol = (GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()
                           + (2.0 / temp) * 2.0 ** -22 * np.abs(v[i]).sum() * cmax)
                    err = np.abs(g[i] - rg[i]).max()
                    assert err <= tol, (temp, i, err, tol)


def test_bcjr_low_temperature_matches_viterbi_codeword(tcq):
    # temp -> 0 recovers the hard code: on sequences whose closest Viterbi
    # decision is at least 1e-3 relative apart, temp 1e-4 leaves the runner-up
    # walks a weight below 2^-50
    s = W.gaussian(16, 47, seq_len=64)
    soft, _ = _bcjr_gpu(tcq, s, 8, 1e-4)
    st, _, margin = oracle.viterbi_f64(s, 8)
    hard = oracle.codebook_f64(8)[st.astype(np.int64)]
    ok = margin > 1e-3
    assert ok.sum() >= 2
    assert np.abs(soft[ok] - hard[ok]).max() <= SOFT_ATOL


# ---------------------------------------------------------------- VJP
@pytest.mark.parametrize("name,temp,nsample", [("l12_gauss1024", 0.05, 12), ("l8_gauss64", 0.1, 64)])
def test_vjp_matches_oracle(tcq, name, temp, nsample):
    w = W.WORKLOADS[name]
    s = W.sequences(name)
    v = np.ones_like(s)                      # gradient of sum of soft codewords
    sd = _dev(s)
    soft, _ = tcq.bcjr_soft(sd, w.L, temp)
    g = tcq.bcjr_soft_backward(sd, w.L, temp, soft, _dev(v))
    torch.cuda.synchronize()
    g = g.cpu().numpy()
    assert np.all(np.isfinite(g))
    idx = np.arange(s.shape[0]) if nsample >= s.shape[0] else \
        np.random.default_rng(5).choice(s.shape[0], nsample, replace=False)
    rg, _ = oracle.bcjr_vjp(s[idx], v[idx], w.L, temp)
    for i, j in enumerate(idx):
        tol = GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()
        assert np.abs(g[j] - rg[i]).max() <= tol, (j, np.abs(g[j] - rg[i]).max(), tol)


@pytest.mark.parametrize("L", [8, 12, 16])
@pytest.mark.parametrize("T,n,temp", [(1, 2, 0.3), (2, 3, 0.3), (5, 9, 0.3), (33, 3, 0.3),
                                      (64, 2, 0.01)])
def test_vjp_edge_shapes_random_cotangent(tcq, L, T, n, temp):
    # ragged batches, short sequences and a low temperature, through both
    # gradient entry points (separate backward and the one-sweep form)
    s = W.gaussian(n, 1300 + T, seq_len=T)
    v = W.gaussian(n, 1400 + T, seq_len=T)
    sd, vd = _dev(s), _dev(v)
    soft, _ = tcq.bcjr_soft(sd, L, temp)
    g1 = tcq.bcjr_soft_backward(sd, L, temp, soft, vd)
    soft2, lz2, g2 = tcq.bcjr_soft_and_grad(sd, L, temp, vd)
    torch.cuda.synchronize()
    rg, rsoft = oracle.bcjr_vjp(s, v, L, temp)
    assert np.abs(soft2.cpu().numpy() - rsoft).max() <= SOFT_ATOL
    for g in (g1.cpu().numpy(), g2.cpu().numpy()):
        for i in range(n):
            tol = GRAD_RTOL_OF_MAX * np.abs(rg[i]).max() + 1e-6
            assert np.abs(g[i] - rg[i]).max() <= tol, (i, np.abs(g[i] - rg[i]).max(), tol)


def test_vjp_l16_rht_block_full(tcq):
    # L = 16 gradient of the sum of soft codewords on the whole 1024 x 1024 RHT
    # block (4,096 sequences, the benchmark's launch); the oracle checks a
    # seeded sample, properties are checked on every sequence
    w = W.WORKLOADS["l16_rht1024_grad"]
    s = W.sequences(w.name)
    temp = w.temps[0]
    sd = _dev(s)
    ones = torch.ones_like(sd)
    soft, lz, g = tcq.bcjr_soft_and_grad(sd, 16, temp, ones)
    soft_sep, lz_sep = tcq.bcjr_soft(sd, 16, temp)
    torch.cuda.synchronize()
    soft, g, soft_sep = soft.cpu().numpy(), g.cpu().numpy(), soft_sep.cpu().numpy()
    assert np.all(np.isfinite(g)) and np.all(np.isfinite(soft))
    assert np.abs(soft - soft_sep).max() <= SOFT_ATOL
    assert np.abs(lz.cpu().numpy() - lz_sep.cpu().numpy()).max() <= 1e-3
    # v = 1: sum_u grad_u = (2/temp) Var(sum_t code(x_t)) >= 0
    assert np.all(g.sum(1) >= -GRAD_RTOL_OF_MAX * np.abs(g).sum(1))
    idx = np.sort(np.random.default_rng(16).choice(s.shape[0], 2, replace=False))
    rg, rsoft = oracle.bcjr_vjp(s[idx], np.ones((2, 256)), 16, temp)
    assert np.abs(soft[idx] - rsoft).max() <= SOFT_ATOL
    for i, j in enumerate(idx):
        tol = GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()
        assert np.abs(g[j] - rg[i]).max() <= tol, (j, np.abs(g[j] - rg[i]).max(), tol)


def test_vjp_random_cotangent_and_autograd(tcq):
    s = W.gaussian(5, 61, seq_len=40)
    v = W.gaussian(5, 62, seq_len=40)
    sd = _dev(s).requires_grad_(True)
    soft = tcq.BcjrSoft.apply(sd, 8, 0.2)
    (soft * _dev(v)).sum().backward()
    g = sd.grad.cpu().numpy()
    rg, _ = oracle.bcjr_vjp(s, v, 8, 0.2)
    for i in range(5):
        assert np.abs(g[i] - rg[i]).max() <= GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()


# ---------------------------------------------------------------- curvature-weighted search
@pytest.mark.parametrize("L,n", [(8, 64), (12, 256), (16, 6)])
def test_weighted_viterbi_bit_exact(tcq, L, n):
    s = W.gaussian(n, 600 + L)
    D = W.curvature(n, 700 + L)
    st, mse = tcq.viterbi_encode(_dev(s), L, D=_dev(D))
    torch.cuda.synchronize()
    st = st.cpu().view(torch.int16).numpy().view(np.uint16)
    rst, rmse, rmg = oracle.map_rows(oracle.viterbi_f32, [s], L, D=D, margin=True)
    assert np.array_equal(st, rst)
    assert np.array_equal(mse.cpu().numpy().view(np.uint32), rmse.view(np.uint32))
    _, _, mg = _viterbi_gpu(tcq, s, L, margin=True, D=D)
    assert _same_f32(mg, rmg)


def test_weighted_full_workload(tcq):
    s = W.sequences("l12_curv1024")
    D = W.weights("l12_curv1024")
    sd, Dd = _dev(s), _dev(D)
    st, mse = tcq.viterbi_encode(sd, 12, D=Dd)
    rst, rmse = oracle.viterbi_f32(s, 12, D=D)
    assert np.array_equal(st.cpu().view(torch.int16).numpy().view(np.uint16), rst)
    assert np.array_equal(mse.cpu().numpy().view(np.uint32), rmse.view(np.uint32))
    soft, lz = tcq.bcjr_soft(sd, 12, 0.05, D=Dd)
    g = tcq.bcjr_soft_backward(sd, 12, 0.05, soft, torch.ones_like(sd), D=Dd)
    torch.cuda.synchronize()
    idx = np.random.default_rng(8).choice(1024, 10, replace=False)
    rg, rsoft = oracle.bcjr_vjp(s[idx], np.ones((10, 256)), 12, 0.05, D=D[idx])
    assert np.abs(soft.cpu().numpy()[idx] - rsoft).max() <= SOFT_ATOL
    gn = g.cpu().numpy()[idx]
    for i in range(10):
        assert np.abs(gn[i] - rg[i]).max() <= GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()
    # the one-sweep form the benchmark times
    soft2, lz2, g2 = tcq.bcjr_soft_and_grad(sd, 12, 0.05, torch.ones_like(sd), D=Dd)
    torch.cuda.synchronize()
    assert np.abs(soft2.cpu().numpy()[idx] - rsoft).max() <= SOFT_ATOL
    assert np.abs(lz2.cpu().numpy() - lz.cpu().numpy()).max() <= 1e-3
    g2n = g2.cpu().numpy()[idx]
    for i in range(10):
        assert np.abs(g2n[i] - rg[i]).max() <= GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()


@pytest.mark.parametrize("L", [8, 12, 16])
def test_weighted_gradient_random_cotangent(tcq, L):
    s = W.gaussian(3, 1800 + L, seq_len=48)
    D = W.curvature(3, 1900 + L, seq_len=48)
    v = W.gaussian(3, 2000 + L, seq_len=48)
    sd, Dd, vd = _dev(s), _dev(D), _dev(v)
    soft, _ = tcq.bcjr_soft(sd, L, 0.2, D=Dd)
    g1 = tcq.bcjr_soft_backward(sd, L, 0.2, soft, vd, D=Dd)
    _, _, g2 = tcq.bcjr_soft_and_grad(sd, L, 0.2, vd, D=Dd)
    torch.cuda.synchronize()
    rg, _ = oracle.bcjr_vjp(s, v, L, 0.2, D=D)
    for g in (g1.cpu().numpy(), g2.cpu().numpy()):
        for i in range(3):
            assert np.abs(g[i] - rg[i]).max() <= GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()


@pytest.mark.parametrize("L", [8, 16])
def test_weighted_bcjr(tcq, L):
    s = W.gaussian(3, 800 + L, seq_len=64)
    D = W.curvature(3, 900 + L, seq_len=64)
    soft, lz = _bcjr_gpu_w(tcq, s, L, 0.2, D)
    rsoft, rlz = oracle.bcjr_soft(s, L, 0.2, D=D)
    assert np.abs(soft - rsoft).max() <= SOFT_ATOL
    assert np.all(np.abs(lz - rlz) <= 1e-5 * np.abs(rlz) + 1e-4)


@pytest.mark.parametrize("L", [12, 16])
@pytest.mark.parametrize("temp", [0.1, 1e-2])
def test_weighted_bcjr_outliers(tcq, L, temp):
    # curvature weights on rows with outliers far outside the code range: the
    # removed per-step terms kappa D_u (r_u - s_u)^2 carry the weight, and the
    # gradient of the fused call is centred on the clamped targets
    s = _outlier_rows(4, 5200 + L)
    D = W.curvature(4, 5300 + L, seq_len=s.shape[1])
    v = W.gaussian(4, 5400 + L, seq_len=s.shape[1])
    soft, lz = _bcjr_gpu_w(tcq, s, L, temp, D)
    _, _, g = tcq.bcjr_soft_and_grad(_dev(s), L, temp, _dev(v), D=_dev(D))
    torch.cuda.synchronize()
    rsoft, rlz = oracle.map_rows(oracle.bcjr_soft, [s], L, temp, D=D)
    rg, _ = oracle.map_rows(oracle.bcjr_vjp, [s, v], L, temp, D=D)
    assert np.abs(soft - rsoft).max() <= SOFT_ATOL
    assert np.all(np.abs(lz - rlz) <= 1e-5 * np.abs(rlz) + 1e-3)
    g = g.cpu().numpy()
    cmax = float(np.abs(oracle.codebook_f32(L)).max())
    for i in range(s.shape[0]):
        # the floor of the extreme-target VJP test; grad_u carries the factor D_u
        tol = (GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()
               + (2.0 / temp) * 2.0 ** -22 * np.abs(v[i]).sum() * cmax * D[i].max())
        assert np.abs(g[i] - rg[i]).max() <= tol


def _bcjr_gpu_w(tcq, s, L, temp, D):
    soft, lz = tcq.bcjr_soft(_dev(s), L, temp, D=_dev(D))
    torch.cuda.synchronize()
    return soft.cpu().numpy(), lz.cpu().numpy()


# ---------------------------------------------------------------- tail-biting encode
def _tb_valid(st, L):
    st = st.astype(np.int64)
    low = (1 << (L - 2)) - 1
    return _is_walk(st, L) & ((st[:, 0] >> 2) == (st[:, -1] & low))


@pytest.mark.parametrize("L,n,T", [(8, 64, 256), (12, 96, 256), (16, 4, 256), (8, 9, 17), (12, 5, 6)])
def test_tailbiting_matches_oracle_algorithm4(tcq, L, n, T):
    s = W.gaussian(n, 1100 + L + T, seq_len=T)
    st, mse = tcq.viterbi_encode_tailbiting(_dev(s), L)
    torch.cuda.synchronize()
    st = st.cpu().view(torch.int16).numpy().view(np.uint16)
    rst, rmse, _ = oracle.viterbi_tailbiting_alg4_f32(s, L)
    assert np.array_equal(st, rst)
    assert np.array_equal(mse.cpu().numpy().view(np.uint32), rmse.view(np.uint32))
    assert np.all(_tb_valid(st, L))


def test_tailbiting_weighted(tcq):
    s = W.gaussian(32, 1201)
    D = W.curvature(32, 1202)
    st, mse = tcq.viterbi_encode_tailbiting(_dev(s), 12, D=_dev(D))
    torch.cuda.synchronize()
    rst, rmse, _ = oracle.viterbi_tailbiting_alg4_f32(s, 12, D=D)
    assert np.array_equal(st.cpu().view(torch.int16).numpy().view(np.uint16), rst)
    assert np.array_equal(mse.cpu().numpy().view(np.uint32), rmse.view(np.uint32))


def test_tailbiting_l16_rht_block_pack_decode(tcq):
    s = W.sequences("l16_rht1024")
    sd = _dev(s)
    st_d, mse_d = tcq.viterbi_encode_tailbiting(sd, 16)
    bits = tcq.pack_states(st_d, 16, tcq.TAILBITING)            # exactly 2 bits per weight
    out = tcq.decode(bits, 16, 256, tcq.TAILBITING, tcq.OUT_TILE16, 1024, 1024)
    torch.cuda.synchronize()
    st = st_d.cpu().view(torch.int16).numpy().view(np.uint16)
    mse = mse_d.cpu().numpy()
    assert bits.shape == (4096, 16)
    assert np.all(_tb_valid(st, 16))
    assert np.array_equal(_seq_mse_f32(s, st, 16).view(np.uint32), mse.view(np.uint32))
    ref = oracle.codebook_f16(16)[st.astype(np.int64)]            # decode = code of the walk
    nr = 1024 // 16
    tiles = out.cpu().numpy().view(np.uint16).reshape(nr, 16, nr, 16).transpose(0, 2, 1, 3).reshape(-1, 256)
    assert np.array_equal(tiles, ref.view(np.uint16))
    idx = np.array([0, 4095, 1234])
    rst, rmse, _ = oracle.viterbi_tailbiting_alg4_f32(s[idx], 16)
    assert np.array_equal(st[idx], rst)
    assert abs(float(mse.mean()) - 0.0697) < 0.004               # page: L=16 tail-biting MSE


# ---------------------------------------------------------------- soft codeword + VJP in one sweep
@pytest.mark.parametrize("name,temp,nsample,weighted", [("l12_gauss1024", 0.05, 12, False),
                                                       ("l8_gauss64", 0.1, 64, True)])
def test_soft_and_grad_one_sweep(tcq, name, temp, nsample, weighted):
    w = W.WORKLOADS[name]
    s = W.sequences(name)
    D = W.curvature(s.shape[0], 31) if weighted else None
    v = W.gaussian(s.shape[0], 32)
    soft, lz, g = tcq.bcjr_soft_and_grad(_dev(s), w.L, temp, _dev(v), D=None if D is None else _dev(D))
    torch.cuda.synchronize()
    soft, lz, g = soft.cpu().numpy(), lz.cpu().numpy(), g.cpu().numpy()
    idx = np.arange(s.shape[0]) if nsample >= s.shape[0] else \
        np.random.default_rng(9).choice(s.shape[0], nsample, replace=False)
    Di = None if D is None else D[idx]
    rg, rsoft = oracle.bcjr_vjp(s[idx], v[idx], w.L, temp, D=Di)
    _, rlz = oracle.bcjr_soft(s[idx], w.L, temp, D=Di)
    assert np.abs(soft[idx] - rsoft).max() <= SOFT_ATOL
    assert np.all(np.abs(lz[idx] - rlz) <= 1e-5 * np.abs(rlz) + 1e-3)
    for i, j in enumerate(idx):
        assert np.abs(g[j] - rg[i]).max() <= GRAD_RTOL_OF_MAX * np.abs(rg[i]).max()


# ---------------------------------------------------------------- random-sign Hadamard rotation
RHT_ATOL = 2e-5      # ~log2(R*C) fp32 rounding steps on partial sums of unit-variance data


def _signs(n, seed):
    return (np.random.default_rng(seed).integers(0, 2, n) * 2 - 1).astype(np.float32)


# every row-pass width (2^11..2^13 in registers, narrower through shared memory)
# and every column-pass split (one pass of <= 10 bits; 5+6, 6+6, 6+7, 7+7 bits)
@pytest.mark.parametrize("R,C", [(1024, 1024), (32, 8192), (8192, 32), (256, 64), (64, 2048),
                                 (32, 4096), (4096, 64), (16384, 32), (2048, 128),
                                 (8192, 1024)])
def test_rht_matches_dense_definition(tcq, R, C):
    W = W_ = np.random.default_rng(R * 3 + C).standard_normal((R, C)).astype(np.float32)
    s1, s2 = _signs(R, R), _signs(C, C + 1)
    out = tcq.rht(_dev(W), _dev(s1), _dev(s2)).cpu().numpy()
    ref = oracle.rht(W_, s1, s2) if R * C <= 1 << 20 and max(R, C) <= 8192 else None
    if ref is None:
        ri = np.random.default_rng(1).choice(R, 6, replace=False)
        ci = np.random.default_rng(2).choice(C, 6, replace=False)
        ref = oracle.rht_entries(W_, s1, s2, ri, ci)
        out = out[ri][:, ci]
    assert np.abs(out - ref).max() <= RHT_ATOL


def test_rht_in_place_and_8192_square_sampled(tcq):
    R = C = 8192
    W = np.random.default_rng(11).standard_t(5, (R, C)).astype(np.float32)
    s1, s2 = _signs(R, 12), _signs(C, 13)
    d = _dev(W)
    tcq.rht(d, _dev(s1), _dev(s2), out=d)                        # in place
    torch.cuda.synchronize()
    got = d.cpu().numpy()
    ri = np.array([0, 1, 4095, 8191])
    ci = np.array([0, 77, 8190])
    ref = oracle.rht_entries(W, s1, s2, ri, ci)
    assert np.abs(got[ri][:, ci] - ref).max() <= 4 * RHT_ATOL * np.sqrt(5 / 3)
    assert abs(float(np.linalg.norm(got.astype(np.float64))) / float(np.linalg.norm(W.astype(np.float64))) - 1) < 1e-5
    # the rotation is orthonormal and (H/sqrt n)^2 = I: rotating the result
    # again with unit signs gives diag(s1) W diag(s2), on all 67 M entries.
    # Each of the 2 x 26 butterfly levels rounds once, at 2^-24 of values that
    # stay within sqrt(2)^26 of the entries' scale only in the worst case;
    # the bound below is 64 roundings of the largest entry.
    tcq.rht(d, _dev(np.ones(R, np.float32)), _dev(np.ones(C, np.float32)), out=d)
    back = d * _dev(s1)[:, None] * _dev(s2)[None, :]
    err = float((back - _dev(W)).abs().max())
    print(f"rht round trip on 8192 x 8192: max |error| {err:.3g}, max |W| {np.abs(W).max():.3g}")
    assert err <= 64 * 2.0 ** -24 * float(np.abs(W).max())


# ---------------------------------------------------------------- decode fused into a GEMV
def _gemv_ref(bits, rows, cols, x, L=16, layout=0, tile_rows=None):
    """fp64 y = W x from the oracle's fp16 decode, and the rigorous fp32
    summation bound (cols + 1) 2^-24 sum_j |W_ij x_j| for each row."""
    nc = cols // 16
    if tile_rows is None:
        Wm = oracle.decode_tiles(bits, rows, cols, L=L, layout=layout).astype(np.float64)
        terms = Wm * x[None, :].astype(np.float64)
        return terms.sum(1), (cols + 1) * 2.0 ** -24 * np.abs(terms).sum(1)
    ys, bs = [], []
    for R in tile_rows:
        blk = oracle.decode_tiles(bits[R * nc:(R + 1) * nc], 16, cols, L=L, layout=layout).astype(np.float64)
        terms = blk * x[None, :].astype(np.float64)
        ys.append(terms.sum(1)); bs.append((cols + 1) * 2.0 ** -24 * np.abs(terms).sum(1))
    return np.concatenate(ys), np.concatenate(bs)


@pytest.mark.parametrize("L,layout,rows,cols", [(16, 0, 256, 512), (8, 1, 96, 160), (12, 0, 1024, 2048),
                                             (12, 1, 32, 16400), (16, 1, 80, 272)])
def test_decode_gemv_matches_oracle(tcq, L, layout, rows, cols):
    # 16400 columns: a row of 1,025 tiles, split into runs that do not divide it
    rng = np.random.default_rng(rows + cols + L)
    n = (rows // 16) * (cols // 16)
    nw = oracle.stream_words(L, 2, 256, layout)
    bits = rng.integers(0, 2 ** 32, (n, nw), dtype=np.uint32)
    x = rng.standard_normal(cols).astype(np.float32)
    y = tcq.decode_gemv(_dev(bits.view(np.int32)).view(torch.uint32), _dev(x), rows, cols, L=L,
                        layout=layout).cpu().numpy()
    ref, bound = _gemv_ref(bits, rows, cols, x, L=L, layout=layout)
    assert np.all(np.abs(y - ref) <= bound + 1e-30)


@pytest.mark.parametrize("case", ["wide_range", "large", "zeros", "tiny"])
def test_decode_gemv_activation_ranges(tcq, case):
    # fp32 activations spanning many decades, far above fp16's range, exactly
    # zero, or far below it: the products stay fp32, so the same bound holds
    rows, cols = 64, 4096
    rng = np.random.default_rng(77)
    bits = rng.integers(0, 2 ** 32, ((rows // 16) * (cols // 16), 16), dtype=np.uint32)
    x = rng.standard_normal(cols)
    if case == "wide_range":
        x = x * 10.0 ** rng.uniform(-4, 5, cols)
    elif case == "large":
        x = x * 1e7
    elif case == "zeros":
        x = np.zeros(cols)
    else:
        x = x * 1e-9
    x = x.astype(np.float32)
    y = tcq.decode_gemv(_dev(bits.view(np.int32)).view(torch.uint32), _dev(x), rows, cols).cpu().numpy()
    ref, bound = _gemv_ref(bits, rows, cols, x)
    assert np.all(np.isfinite(y))
    assert np.all(np.abs(y - ref) <= bound + 1e-30)


def test_decode_gemv_8192_square_sampled_rows(tcq):
    bits = W.streams("l16_decode_8192sq")
    x = np.random.default_rng(8).standard_normal(8192).astype(np.float32)
    y = tcq.decode_gemv(_dev(bits.view(np.int32)).view(torch.uint32), _dev(x), 8192, 8192).cpu().numpy()
    trs = [0, 1, 255, 511]
    ref, bound = _gemv_ref(bits, 8192, 8192, x, tile_rows=trs)
    got = np.concatenate([y[16 * R:16 * R + 16] for R in trs])
    assert np.all(np.abs(got - ref) <= bound)
