"""The N>1 path on CPU: two gloo ranks.  Sequences are independent, so a
matrix workload is split by 16 x 16-tile rows and a Gaussian batch by
sequences (no data-path collective); the step time is reduced as the maximum
over ranks.  The per-rank work here is the CPU oracle on a tiny slice, since
the CUDA path needs a GPU; what is checked is the host logic bench.py uses:
the ranks' shares are disjoint, cover the workload and are the tiles the
matrix layout says (QTIP blog, "What it buys end to end": one 16 x 16 tile
is one 256-weight sequence)."""
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
    res = {}
    for name in ("l12_gauss1024", "l16_rht1024", "l16_studentt_2048x8192"):
        w = W.WORKLOADS[name]
        batch = bench.rank_batch(w, rank, world)
        lo, hi = bench.shard(w, rank, world)
        # each rank "encodes" the first 2 sequences of its share
        st, mse = oracle.viterbi_f32(batch[:2, :32], 8)
        res[name] = (lo, hi, batch.shape, batch[:2, :4].tolist(), mse.tolist())
    fake_ms = 1.0 + rank                       # rank 1 is the slower one
    job_ms = bench.max_over_ranks(fake_ms, dist, torch.device("cpu"))
    gathered = [None] * world
    dist.all_gather_object(gathered, res)
    out[rank] = (job_ms, gathered)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_split_host_logic():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    import bench
    import tcq_workloads as W
    for r in range(world):
        job_ms, gathered = out[r]
        assert job_ms == 2.0                   # the maximum over ranks
        assert gathered == out[0][1]           # every rank sees the same gathered view
    g = out[0][1]
    for name in ("l12_gauss1024", "l16_rht1024", "l16_studentt_2048x8192"):
        w = W.WORKLOADS[name]
        full = W.sequences(name)
        ranges = [g[r][name][:2] for r in range(world)]
        # disjoint, in order, and covering every sequence
        assert ranges[0][0] == 0 and ranges[-1][1] == w.n_seq
        assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
        for r in range(world):
            lo, hi, shape, head, _ = g[r][name]
            assert tuple(shape) == (hi - lo, 256)
            assert np.array_equal(np.array(head, dtype=np.float32), full[lo:lo + 2, :4])
        if w.rows:
            # whole tile rows: rank r's share is rows [16 a, 16 b) of the matrix
            per_row = w.cols // 16
            assert all(lo % per_row == 0 and hi % per_row == 0 for lo, hi in ranges)
    # strong scaling: the job's units are the workload's, whatever the rank count
    assert bench.scaling_of(W.WORKLOADS["l16_studentt_2048x8192"], 2) == "strong"


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shares_partition_every_workload(world):
    import bench
    import tcq_workloads as W
    for name, w in W.WORKLOADS.items():
        ranges = [bench.shard(w, r, world) for r in range(world)]
        if ranges[0] is None:                  # a replica per rank: the rotation
            assert w.ops == ("rht",)
            assert bench.scaling_of(w, world) == "weak"
            continue
        assert ranges[0][0] == 0 and ranges[-1][1] == w.n_seq
        assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
        assert all(lo <= hi for lo, hi in ranges)


def test_tile_rows_of_a_share_are_the_matrix_rows():
    # the sequences of a rank's share, put back as tiles, are the matrix rows
    # [16 a, 16 b) of the block (tiles_to_sequences is row-major over tiles)
    import bench
    import tcq_workloads as W
    w = W.WORKLOADS["l16_studentt_2048x8192"]
    m = W.student_t_block(w.seed, w.rows, w.cols)
    lo, hi = bench.shard(w, 1, 4)
    share = bench.rank_batch(w, 1, 4)
    a, b = lo // (w.cols // 16), hi // (w.cols // 16)
    assert np.array_equal(share, W.tiles_to_sequences(m[16 * a:16 * b]))


def test_weak_mode_gives_each_gaussian_rank_its_own_batch():
    import bench
    import tcq_workloads as W
    w = W.WORKLOADS["l12_gauss1024"]
    a, b = bench.rank_batch(w, 0, 2, weak=True), bench.rank_batch(w, 1, 2, weak=True)
    assert a.shape == b.shape == (w.n_seq, 256) and a.dtype == np.float32
    assert not np.array_equal(a, b)
    assert np.array_equal(a, W.sequences(w.name))
    assert bench.scaling_of(w, 2, weak=True) == "weak"
