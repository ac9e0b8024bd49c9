"""Host-side bookkeeping of bench.py that runs without a GPU: the oracle
tasks of the CPU baseline and the reference arm, and what each credits."""
import numpy as np

import bench
import tcq_workloads as W


def test_tasks_credit_whole_sequences():
    # a BCJR-only workload at three temperatures splits each sequence into
    # one task per temperature, each credited a third of its 256 weights;
    # any other workload runs one sequence through every step per task
    w = W.WORKLOADS["l16_studentt_2048x8192"]
    tasks = bench._tasks_for(w, 9)
    assert [t[0] for t in tasks] == [0, 0, 0, 1, 1, 1, 2, 2, 2]
    assert [t[1] for t in tasks] == [(1.0,), (0.1,), (0.01,)] * 3
    assert abs(sum(t[2] for t in tasks) - 3 * 256) < 1e-9
    w2 = W.WORKLOADS["l12_gauss1024"]
    tasks = bench._tasks_for(w2, 4, offset=7)
    assert [t[0] for t in tasks] == [7, 8, 9, 10] and all(t[1] is None and t[2] == 256 for t in tasks)


def test_oracle_threads_bounded_by_memory_and_cores():
    import oracle
    for name in ("l8_gauss64", "l12_gauss1024", "l16_studentt_2048x8192", "l16_rht1024_grad"):
        t = bench.oracle_threads(W.WORKLOADS[name])
        assert 1 <= t <= oracle.host_threads()
    # the fp64 tables one L = 16 gradient task holds: alpha, beta, phi, psi
    assert bench._task_bytes(W.WORKLOADS["l16_rht1024_grad"]) == 4 * (1 << 16) * 256 * 8


def test_run_tasks_matches_sequential_oracle():
    # the thread pool runs the same oracle calls as a sequential loop
    w = W.WORKLOADS["l8_gauss64"]
    s = W.sequences(w.name, n_limit=6)
    credit = bench._run_tasks(w, s, None, bench._tasks_for(w, 6), 3)
    assert credit == 6 * 256


def test_metric_and_dtype_labels():
    assert bench._dtype_for(W.WORKLOADS["l16_decode_8192sq"]) == "f16"
    assert bench._dtype_for(W.WORKLOADS["l16_studentt_2048x8192"]) == "f32"
    assert "BCJR soft x3 temps" in bench._metric_for(W.WORKLOADS["l16_studentt_2048x8192"])
    assert bench.DEFAULT_WORKLOAD == "l16_studentt_2048x8192"
    assert set(bench.COMPANIONS) == {"l8_gauss64", "l12_gauss1024", "l16_rht1024", "l16_decode_8192sq"}
