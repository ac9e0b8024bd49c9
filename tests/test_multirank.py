"""The N>1 path on CPU: two gloo ranks, each encoding its own batch (weak
scaling, no data-path collective), with the step time reduced as the maximum
over ranks.  The per-rank work here is the CPU oracle on a tiny slice, since
the CUDA path needs a GPU; what is checked is the host logic bench.py uses."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    import oracle
    import tcq_workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w = W.WORKLOADS["l12_gauss1024"]
    batch = bench.rank_batch(w, rank)
    # each rank "encodes" the first 2 sequences of its own batch
    st, mse = oracle.viterbi_f32(batch[:2, :32], 8)
    fake_ms = 1.0 + rank                       # rank 1 is the slower one
    job_ms = bench.max_over_ranks(fake_ms, dist, torch.device("cpu"))
    gathered = [None] * world
    dist.all_gather_object(gathered, (batch[:2, :4].tolist(), mse.tolist()))
    out[rank] = (job_ms, gathered)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_host_logic():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    import bench
    import tcq_workloads as W
    w = W.WORKLOADS["l12_gauss1024"]
    for r in range(world):
        job_ms, gathered = out[r]
        assert job_ms == 2.0                   # the maximum over ranks
        # every rank sees the same gathered view
        assert gathered == out[0][1]
    g = out[0][1]
    b0 = bench.rank_batch(w, 0)
    assert np.allclose(np.array(g[0][0]), b0[:2, :4])          # rank 0 = the workload itself
    assert not np.allclose(np.array(g[1][0]), b0[:2, :4])      # rank 1: its own batch
    assert np.array_equal(bench.rank_batch(w, 1), bench.rank_batch(w, 1))   # deterministic
    # weak scaling: total units = per-rank units x ranks
    assert w.n_seq * 256 * world == 2 * 262144


def test_rank_batches_for_every_workload_kind():
    import bench
    import tcq_workloads as W
    for name in ("l8_gauss64", "l12_gauss1024"):
        w = W.WORKLOADS[name]
        a, b = bench.rank_batch(w, 0), bench.rank_batch(w, 3)
        assert a.shape == b.shape == (w.n_seq, 256) and a.dtype == np.float32
        assert not np.array_equal(a, b)
