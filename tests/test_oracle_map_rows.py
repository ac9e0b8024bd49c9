"""oracle.map_rows, the thread pool the GPU tests use to compute references:
its results must equal one direct call of the routine, in the same row order,
for every way of cutting the rows (array and keyword inputs, tuple outputs)."""
import numpy as np
import pytest

import oracle
import tcq_workloads as W


@pytest.mark.parametrize("threads", [1, 3, 7, 64])
def test_viterbi_rows_match_direct_call(threads):
    s = W.gaussian(13, 501, seq_len=24)
    D = W.curvature(13, 502, seq_len=24)
    st, mse, mg = oracle.viterbi_f32(s, 8, D=D, margin=True)
    st2, mse2, mg2 = oracle.map_rows(oracle.viterbi_f32, [s], 8, threads=threads, D=D, margin=True)
    assert np.array_equal(st, st2)
    assert np.array_equal(mse.view(np.uint32), mse2.view(np.uint32))
    assert np.array_equal(mg.view(np.uint32), mg2.view(np.uint32))


@pytest.mark.parametrize("threads", [2, 5])
def test_bcjr_rows_match_direct_call(threads):
    s = W.gaussian(6, 503, seq_len=20)
    v = W.gaussian(6, 504, seq_len=20)
    soft, lz = oracle.bcjr_soft(s, 8, 0.3)
    soft2, lz2 = oracle.map_rows(oracle.bcjr_soft, [s], 8, 0.3, threads=threads)
    assert np.array_equal(soft, soft2) and np.array_equal(lz, lz2)
    g, sf = oracle.bcjr_vjp(s, v, 8, 0.3)
    g2, sf2 = oracle.map_rows(oracle.bcjr_vjp, [s, v], 8, 0.3, threads=threads)
    assert np.array_equal(g, g2) and np.array_equal(sf, sf2)
