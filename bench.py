"""Throughput of the bitshift-trellis hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of synthetic input.
The default workload is the largest one that fits a GPU: the BCJR soft
codeword at temperatures 1, 0.1 and 0.01 over a 2048 x 8192 Student-t (nu = 5)
weight block cut into 65,536 sequences of 256 (16 x 16 tiles) on the L = 16
trellis.  The same run measures the four other configurations (L = 8 Viterbi
+ BCJR on 64 Gaussian sequences; L = 12 Viterbi + pack + decode + BCJR soft
and gradient on 1,024; L = 16 Viterbi on the 1024 x 1024 rotated block; the
8192 x 8192 decode) and carries them in the line under ``per_workload``.
The metric is weights per second (whole job, all ranks).

Multi-GPU: sequences are independent, so a matrix workload is split by
16 x 16-tile rows across ranks and a Gaussian batch by sequences (strong
scaling, no data-path collective; ``--weak`` gives every Gaussian rank its
own batch instead).  The rotation runs one replica per rank.  The step time
is the maximum over ranks of the CUDA-event time.

A batch that under-fills the GPU (the 64-sequence L=8 workload) runs its
independent calls (Viterbi and one soft pass per temperature) on separate
streams, each with its own workspace; every other workload runs on one stream.

L2 is flushed before every timed step, outside the step's event pair: a
256 MiB write, then a 256 MiB read of another buffer, which evicts the
write's dirty lines so that the timed kernels do not pay for writing them
back; a ~1 ms device spin follows, so that the step's launches are queued
before the GPU reaches its first event.  `--impl reference` times the plain
CPU oracle on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import tcq_workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "l16_studentt_2048x8192"
# measured in the same run as the default workload and carried in its line
COMPANIONS = ("l8_gauss64", "l12_gauss1024", "l16_rht1024", "l16_decode_8192sq")
NEAR_TIE = 1e-6


def _args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-companions", action="store_true",
                   help="measure only --workload, not the other configurations")
    p.add_argument("--weak", action="store_true",
                   help="Gaussian workloads: every rank encodes its own batch (weak scaling)")
    p.add_argument("--n-seq", type=int, default=0,
                   help="encode only the first N sequences of the workload (profiling runs)")
    return p.parse_args(argv)


def _metric_for(w: W.Workload) -> str:
    if w.ops == ("gemv",):
        return "decoded weights/sec in a batch-1 GEMV (2-bit stream decoded in registers)"
    if w.ops == ("rht",):
        return "rotated weights/sec (random-sign Hadamard rotation, both sides, fp32)"
    if w.ops == ("decode",):
        return "decoded weights/sec (2-bit tail-biting stream -> fp16, 16x16 tiles)"
    parts = []
    if "viterbi" in w.ops:
        parts.append("Viterbi")
    if "viterbi_tb" in w.ops:
        parts.append("tail-biting Viterbi (two-run)")
    if "pack_decode" in w.ops:
        parts.append("pack + decode")
    if "bcjr" in w.ops:
        parts.append("BCJR soft" + (f" x{len(w.temps)} temps" if len(w.temps) > 1 else ""))
    if "bcjr_grad" in w.ops:
        parts.append("BCJR gradient")
    tail = ", curvature-weighted" if w.curv_seed else ""
    return "weights quantized/sec (" + " + ".join(parts) + tail + ")"


def _dtype_for(w: W.Workload) -> str:
    # the type the path computes in: decode forms the fp32 code from integer
    # windows and writes it rounded to fp16; everything else is fp32
    return "f16" if w.ops == ("decode",) else "f32"


# ------------------------------------------------------------------ ranks
def _tiled(w: W.Workload) -> bool:
    return w.rows > 0 and w.cols > 0 and w.ops != ("rht",)


def shard(w: W.Workload, rank: int, world: int, weak: bool = False):
    """Sequence range [lo, hi) of the workload that rank encodes, or None
    when every rank runs a whole replica of its own (the rotation, whose
    column transform mixes all rows, and Gaussian batches under --weak).
    A matrix workload is split by 16 x 16-tile rows (sequence r * (cols/16) + c
    is the tile at (16 r, 16 c)), a Gaussian batch by sequences."""
    if w.ops == ("rht",) or (weak and w.kind == "gaussian" and world > 1):
        return None
    if _tiled(w):
        R, per_row = w.rows // 16, w.cols // 16
        return (rank * R // world) * per_row, ((rank + 1) * R // world) * per_row
    return rank * w.n_seq // world, (rank + 1) * w.n_seq // world


def scaling_of(w: W.Workload, world: int, weak: bool = False) -> str:
    return "weak" if shard(w, 0, max(world, 2), weak) is None else "strong"


def rank_batch(w: W.Workload, rank: int, world: int = 1, weak: bool = False) -> np.ndarray:
    """The input rank `rank` encodes: its share of the workload (see
    ``shard``), or, for a replica, the workload itself on rank 0 and a draw of
    the same distribution from seed + 1000 * rank on the others."""
    rng_seed = w.seed + 1000 * rank
    rg = shard(w, rank, world, weak)
    if w.ops == ("rht",):
        return W.student_t_block(rng_seed, w.rows, w.cols)
    if rg is None:                                   # weak Gaussian replica
        if rank == 0:
            return W.sequences(w.name, n_limit=w.n_seq)
        return np.random.default_rng(rng_seed).standard_normal((w.n_seq, W.SEQ_LEN)).astype(np.float32)
    lo, hi = rg
    if w.ops in (("decode",), ("gemv",)):
        return np.ascontiguousarray(W.bitstream(w.n_seq, w.seed)[lo:hi])
    return np.ascontiguousarray(W.sequences(w.name)[lo:hi])


def rank_weights(w: W.Workload, rank: int, world: int = 1, weak: bool = False):
    D = W.weights(w.name)
    if D is None:
        return None
    rg = shard(w, rank, world, weak)
    return D if rg is None else np.ascontiguousarray(D[rg[0]:rg[1]])


def max_over_ranks(value: float, dist, device) -> float:
    """Step time of the job = the slowest rank's (a timing collective only)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples the SM clock and the clock-event reasons (read-only NVML queries)
    from a background thread while the timed region runs, plus once on entry
    and once on exit so that even a sub-millisecond region gets samples."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown"}

    def __init__(self, gpu_uuid: str):
        self.gpu_uuid = gpu_uuid
        self.samples = []
        self.max_mhz = None
        self._stop = None

    def _sample(self):
        import pynvml
        sm = pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        try:
            rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            rs = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((sm, rs))

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._sample()
        except Exception:
            self.h = None
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.wait(0.01):
                try:
                    self._sample()
                except Exception:
                    return
        self._t = threading.Thread(target=loop, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=2)
            try:
                self._sample()
            except Exception:
                pass

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        reasons = sorted({name for _, rs in self.samples for bit, name in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU oracle
def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_seq(w: W.Workload, s: np.ndarray, D=None, temps=None) -> None:
    """The oracle's pass over one or more sequences (rows of s); ``temps``
    narrows the soft passes of a BCJR-only workload to some temperatures."""
    import oracle
    if "viterbi" in w.ops:
        st, _ = oracle.viterbi_f32(s, w.L, D=D)
        if "pack_decode" in w.ops:
            oracle.decode(oracle.pack(st, w.L, oracle.FREE_START), w.L, s.shape[1], oracle.FREE_START)
    if "viterbi_tb" in w.ops:
        oracle.viterbi_tailbiting_alg4_f32(s, w.L, D=D)
    for temp in (w.temps if temps is None else temps):
        if "bcjr_grad" in w.ops and temp == w.temps[0]:
            oracle.bcjr_vjp(s, np.ones_like(s, dtype=np.float64), w.L, temp, D=D)  # also yields soft
        elif "bcjr" in w.ops:
            oracle.bcjr_soft(s, w.L, temp, D=D)


def _oracle_streams(bits: np.ndarray, w: W.Workload) -> None:
    import oracle
    if w.ops == ("gemv",):          # whole bands of tile-rows: decode, then the matvec
        nc = w.cols // 16
        bands = bits.shape[0] // nc
        x = W.gemv_vector(w.name).astype(np.float64)
        oracle.decode_tiles(bits[: bands * nc], 16 * bands, w.cols, L=w.L).astype(np.float64) @ x
        return
    oracle.decode(bits, w.L, 256, oracle.TAILBITING)


_RHT_SAMPLE = (256, 1024)     # leading block the oracle rotates by its dense definition


def _oracle_rht_sample(w: W.Workload) -> int:
    """Dense-definition rotation of the leading 256 x 1024 block of the
    workload's matrix (its own 256- and 1024-point transforms); returns the
    weights rotated."""
    import oracle
    Wm, s1, s2 = W.rotation_input(w.name)
    r, c = _RHT_SAMPLE
    oracle.rht(Wm[:r, :c], s1[:r], s2[:c])
    return r * c


def _task_bytes(w: W.Workload) -> int:
    """Host memory one oracle task holds at once (the fp64 per-step tables)."""
    n = (1 << w.L) * W.SEQ_LEN * 8
    if "bcjr_grad" in w.ops:
        return 4 * n
    if "bcjr" in w.ops or "viterbi" in w.ops or "viterbi_tb" in w.ops:
        return 2 * n
    return 64 << 20


def oracle_threads(w: W.Workload) -> int:
    """Threads for the multi-core oracle run: every usable host core, bounded
    so that the tasks' tables fit in the memory available."""
    import oracle
    cores = oracle.host_threads()
    try:
        import psutil
        avail = psutil.virtual_memory().available
        cores = min(cores, max(1, int(avail * 0.5 // _task_bytes(w))))
    except Exception:
        pass
    return max(1, cores)


def _tasks_for(w: W.Workload, n_tasks: int, offset: int = 0):
    """(sequence index, temps or None, weight credit) of n_tasks oracle tasks:
    a BCJR-only workload with several temperatures splits each sequence into
    one task per temperature (credit 1/len(temps) of its 256 weights)."""
    split = w.ops == ("bcjr",) and len(w.temps) > 1
    out = []
    for j in range(offset, offset + n_tasks):
        if split:
            out.append((j // len(w.temps), (w.temps[j % len(w.temps)],), W.SEQ_LEN / len(w.temps)))
        else:
            out.append((j, None, float(W.SEQ_LEN)))
    return out


def _run_tasks(w, s, D, tasks, threads):
    from concurrent.futures import ThreadPoolExecutor

    def one(task):
        i, temps, _ = task
        _oracle_seq(w, s[i:i + 1], None if D is None else D[i:i + 1], temps)

    if threads == 1:
        for t in tasks:
            one(t)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, tasks))
    return sum(t[2] for t in tasks)


def cpu_baseline(w: W.Workload, budget_s: float = 10.0) -> dict:
    """Time the oracle, as it stands, on a bounded sample of the workload:
    single-threaded, then over every usable host core (a thread pool over
    sequences: the C routines run without the GIL).  ``value`` is the
    all-cores rate; the single-thread rate rides along."""
    import oracle
    oracle.build()
    host = {"cpu_model": _cpu_model(), "host_cores": os.cpu_count(), "usable_cores": oracle.host_threads()}
    if w.ops == ("rht",):
        done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < 2.0:
            done += _oracle_rht_sample(w)
        dt = time.perf_counter() - t0
        return {"value": done / dt, "unit": "weights/s", "cores": os.cpu_count(), "kind": "oracle",
                "sample": f"dense-definition rotation of the leading {_RHT_SAMPLE[0]} x "
                          f"{_RHT_SAMPLE[1]} block of {w.name} (numpy matmul, all BLAS threads), "
                          f"{dt:.1f} s wall", "host": host}
    if w.ops in (("decode",), ("gemv",)):
        bits = W.streams(w.name)
        chunk = 1024 if w.ops == ("decode",) else w.cols // 16 * 8
        n_done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < budget_s and n_done + chunk <= bits.shape[0]:
            _oracle_streams(bits[n_done:n_done + chunk], w)
            n_done += chunk
        dt = time.perf_counter() - t0
        return {"value": n_done * W.SEQ_LEN / dt, "unit": "weights/s", "cores": 1, "kind": "oracle",
                "sample": f"first {n_done} of {w.n_seq} streams of {w.name} (numpy), {dt:.1f} s wall",
                "host": host}
    threads = oracle_threads(w)
    n_avail = min(w.n_seq, 4096)
    s = W.sequences(w.name, n_limit=n_avail)
    D = W.weights(w.name, n_limit=n_avail)
    max_tasks = n_avail * (len(w.temps) if w.ops == ("bcjr",) and len(w.temps) > 1 else 1)
    # single thread: tasks one at a time until half the budget is spent
    done_w, n_t, t0 = 0.0, 0, time.perf_counter()
    while (time.perf_counter() - t0 < budget_s / 2 or n_t == 0) and n_t < max_tasks:
        done_w += _run_tasks(w, s, D, _tasks_for(w, 1, n_t), 1)
        n_t += 1
    dt1 = time.perf_counter() - t0
    single = {"value": done_w / dt1, "cores": 1,
              "sample": f"{n_t} oracle tasks ({_task_desc(w)}) of {w.name}, {dt1:.1f} s wall"}
    # all cores: about half the budget's worth of tasks, `threads` at a time
    per_task = dt1 / n_t
    want = int(budget_s / 2 / max(per_task, 1e-9)) * threads
    n_tasks = min(max(threads, want), max_tasks)
    t0 = time.perf_counter()
    done_w = _run_tasks(w, s, D, _tasks_for(w, n_tasks), threads)
    dtm = time.perf_counter() - t0
    return {"value": done_w / dtm, "unit": "weights/s", "cores": threads, "kind": "oracle",
            "sample": f"{n_tasks} oracle tasks ({_task_desc(w)}) of {w.name} on {threads} threads, "
                      f"{dtm:.1f} s wall",
            "single_thread": single, "host": host}


def _task_desc(w: W.Workload) -> str:
    if w.ops == ("bcjr",) and len(w.temps) > 1:
        return "one sequence at one temperature each"
    return "one sequence through every step each"


def run_reference(a) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = W.WORKLOADS[a.workload]
    import oracle
    oracle.build()
    line_base = {
        "impl": "reference", "metric": _metric_for(w), "unit": "weights/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "higher_is_better": True,
        "scaling": scaling_of(w, a.gpus, a.weak), "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
    }
    host = {"cpu_model": _cpu_model(), "host_cores": os.cpu_count(), "usable_cores": oracle.host_threads()}
    if w.ops == ("rht",):
        times = []
        for i in range(a.warmup + a.steps):
            t0 = time.perf_counter()
            done = _oracle_rht_sample(w)
            if i >= a.warmup:
                times.append(time.perf_counter() - t0)
        step_s = sum(times) / len(times)
        value = done / step_s
        print(json.dumps({**line_base, "value": value, "ms_per_step": step_s * 1e3,
                          "config": {"workload": w.name, "rows": w.rows, "cols": w.cols},
                          "cpu_baseline": {"value": value, "unit": "weights/s", "cores": os.cpu_count(),
                                           "kind": "oracle", "sample": "leading 256 x 1024 block per step",
                                           "host": host},
                          "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return
    times, credit = [], 0.0
    if w.ops in (("decode",), ("gemv",)):
        per_step = 1024 if w.ops == ("decode",) else w.cols // 16 * 4
        data = W.streams(w.name)
        threads = 1
        for i in range(a.warmup + a.steps):
            lo = (i * per_step) % (data.shape[0] - per_step + 1)
            t0 = time.perf_counter()
            _oracle_streams(data[lo:lo + per_step], w)
            if i >= a.warmup:
                times.append(time.perf_counter() - t0)
        credit = per_step * W.SEQ_LEN
        sample = f"{per_step} streams per step of {w.name} (numpy)"
    else:
        # each step: one round of concurrent oracle tasks, one per thread
        threads = oracle_threads(w)
        n_tasks = threads
        n_seq_needed = len({t[0] for t in _tasks_for(w, n_tasks)})
        s = W.sequences(w.name, n_limit=min(w.n_seq, n_seq_needed))
        D = W.weights(w.name, n_limit=min(w.n_seq, n_seq_needed))
        tasks = _tasks_for(w, n_tasks)
        for i in range(a.warmup + a.steps):
            t0 = time.perf_counter()
            credit = _run_tasks(w, s, D, tasks, threads)
            if i >= a.warmup:
                times.append(time.perf_counter() - t0)
        sample = f"{n_tasks} oracle tasks per step ({_task_desc(w)}) of {w.name} on {threads} threads"
    step_s = sum(times) / len(times)
    value = credit / step_s
    print(json.dumps({
        **line_base, "value": value, "ms_per_step": step_s * 1e3,
        "config": {"workload": w.name, "L": w.L, "n_seq": w.n_seq, "seq_len": W.SEQ_LEN,
                   "temps": list(w.temps)},
        "cpu_baseline": {"value": value, "unit": "weights/s", "cores": threads, "kind": "oracle",
                         "sample": sample, "host": host},
        "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ------------------------------------------------------------------ GPU arm
class Ctx:
    """Per-process GPU state shared by the measurements of one run."""

    def __init__(self, a):
        import torch
        import trellis_coded_weight_bitshift_b200 as tcq
        from trellis_coded_weight_bitshift_b200.build import build
        self.torch, self.tcq, self.a = torch, tcq, a
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        self.dist = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
            self.dist = dist
        else:
            torch.cuda.set_device(0)
        if self.rank == 0:
            build()
        if self.dist is not None:
            self.dist.barrier()
        self.dev = torch.device("cuda", torch.cuda.current_device())
        self.stream = torch.cuda.current_stream()
        self.flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=self.dev)
        self.flush_r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=self.dev)
        uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
        self.gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid

    def flush_l2(self):
        self.flush.fill_(1)                                  # every line of L2 replaced ...
        self.flush_r.sum()                                   # ... and the dirty ones written back
        # keep the GPU busy for ~1 ms more, so that the step's first event and
        # launches are queued before the GPU reaches them: the events then time
        # the kernels, not the host's Python call overhead
        self.torch.cuda._sleep(2_000_000)

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()


def measure(ctx: Ctx, w: W.Workload, steps: int, warmup: int, e2e_steps: int, weak: bool) -> dict:
    """Time `steps` steps of workload w (after `warmup`), then the same step
    end to end from pinned host memory; return the measurement record."""
    torch, tcq, dev, stream = ctx.torch, ctx.tcq, ctx.dev, ctx.stream
    rank, world, dist = ctx.rank, ctx.world, ctx.dist
    rg = shard(w, rank, world, weak)
    n_local = w.n_seq if rg is None else rg[1] - rg[0]
    rows_local = w.rows if (rg is None or not _tiled(w)) else (rg[1] - rg[0]) // (w.cols // 16) * 16
    host = rank_batch(w, rank, world, weak)
    as_words = w.ops in (("decode",), ("gemv",))
    x = (torch.from_numpy(host.view(np.int32)).to(dev).view(torch.uint32) if as_words
         else torch.from_numpy(host).to(dev))
    h2d_bytes = host.nbytes
    if w.ops == ("gemv",):
        xvec = torch.from_numpy(W.gemv_vector(w.name)).to(dev)
        yvec = torch.empty((rows_local,), dtype=torch.float32, device=dev)
    if w.ops == ("rht",):
        _, s1h, s2h = W.rotation_input(w.name)
        sr, sc = torch.from_numpy(s1h).to(dev), torch.from_numpy(s2h).to(dev)
        rot_out = torch.empty_like(x)
    ws_v = ws_b = ws_g = None
    if "viterbi" in w.ops or "viterbi_tb" in w.ops:
        ws_v = torch.empty(tcq.viterbi_workspace_size(w.L, 256, n_local), dtype=torch.uint8, device=dev)
    if "bcjr" in w.ops and not ("bcjr_grad" in w.ops and len(w.temps) == 1):
        ws_b = torch.empty(tcq.bcjr_workspace_size(w.L, 256, n_local), dtype=torch.uint8, device=dev)
    if "bcjr_grad" in w.ops:
        ws_g = torch.empty(tcq.bcjr_workspace_size(w.L, 256, n_local, True), dtype=torch.uint8, device=dev)
    # a batch that under-fills the GPU runs its independent calls (Viterbi, one
    # soft pass per temperature) on separate streams, each with its own workspace
    concurrent = w.concurrent and "bcjr_grad" not in w.ops and "pack_decode" not in w.ops
    side = [torch.cuda.Stream(device=dev) for _ in range(1 + len(w.temps))] if concurrent else []
    ws_bt = ([torch.empty(tcq.bcjr_workspace_size(w.L, 256, n_local), dtype=torch.uint8, device=dev)
              for _ in w.temps] if concurrent and "bcjr" in w.ops else [])
    ones = (torch.ones((n_local, W.SEQ_LEN), dtype=torch.float32, device=dev)
            if "bcjr_grad" in w.ops else None)
    wts = rank_weights(w, rank, world, weak)
    Dd = torch.from_numpy(wts).to(dev) if wts is not None else None

    kern_ms: dict[str, list[float]] = {}
    launches_per_step = 0

    def step(inp, timed: bool):
        nonlocal launches_per_step
        outs, ev, spans = [], [], []
        n_launch = 0

        def mark(name):
            if timed:
                e = torch.cuda.Event(enable_timing=True)
                e.record(stream)
                ev.append((name, e))

        if w.ops == ("gemv",):
            mark("start")
            outs.append(tcq.decode_gemv(inp, xvec, rows_local, w.cols, L=w.L, out=yvec))
            mark("decode_gemv")
            n_launch += 1
        elif w.ops == ("rht",):
            mark("start")
            outs.append(tcq.rht(inp, sr, sc, out=rot_out))
            mark("rht")
            n_launch += 3
        elif w.ops == ("decode",):
            mark("start")
            outs.append(tcq.decode(inp, w.L, 256, tcq.TAILBITING, tcq.OUT_TILE16, rows_local, w.cols))
            mark("decode_tile16")
            n_launch += 1
        elif concurrent:
            mark("start")
            jobs = []
            if "viterbi" in w.ops:
                jobs.append(("viterbi", lambda: list(tcq.viterbi_encode(inp, w.L, ws_v, D=Dd)), 2))
            if "bcjr" in w.ops:
                for i, temp in enumerate(w.temps):
                    jobs.append((f"bcjr_soft_t{temp:g}",
                                 lambda t=temp, ws=ws_bt[i]: list(tcq.bcjr_soft(inp, w.L, t, ws, D=Dd)), 1))
            for (name, fn, nl), sst in zip(jobs, side):
                sst.wait_stream(stream)
                with torch.cuda.stream(sst):
                    e0 = torch.cuda.Event(enable_timing=True)
                    e0.record(sst)
                    outs += fn()
                    e1 = torch.cuda.Event(enable_timing=True)
                    e1.record(sst)
                spans.append((name, e0, e1))
                n_launch += nl
            for sst in side[:len(jobs)]:
                stream.wait_stream(sst)
            mark("end")
        else:
            mark("start")
            if "viterbi" in w.ops:
                st, mse = tcq.viterbi_encode(inp, w.L, ws_v, D=Dd)
                mark("viterbi")
                n_launch += 2
                outs += [st, mse]
                if "pack_decode" in w.ops:
                    bits = tcq.pack_states(st, w.L, tcq.FREE_START)
                    dec = tcq.decode(bits, w.L, W.SEQ_LEN, tcq.FREE_START, tcq.OUT_SEQ)
                    mark("pack_decode_seq")
                    n_launch += 2
                    outs.append(dec)
            if "viterbi_tb" in w.ops:
                st, mse = tcq.viterbi_encode_tailbiting(inp, w.L, ws_v, D=Dd)
                mark("viterbi_tb")
                n_launch += 4
                outs += [st, mse]
            for i, temp in enumerate(w.temps):
                if "bcjr_grad" in w.ops and i == 0:
                    # the cotangent (gradient of the sum of soft codewords) is
                    # known up front: one sweep gives soft, log Z and grad
                    soft, lz, g = tcq.bcjr_soft_and_grad(inp, w.L, temp, ones, ws_g, D=Dd)
                    mark(f"bcjr_soft_vjp_t{temp:g}")
                    n_launch += 1
                    outs += [soft, lz, g]
                    continue
                soft, lz = tcq.bcjr_soft(inp, w.L, temp, ws_b, D=Dd)
                mark(f"bcjr_soft_t{temp:g}")
                n_launch += 1
                outs += [soft, lz]
        launches_per_step = n_launch
        return outs, ev, spans

    for _ in range(warmup):
        step(x, False)
    torch.cuda.synchronize()

    # ---- device-timed region ----
    ctx.barrier()
    torch.cuda.synchronize()
    step_ms = []
    with ClockSampler(ctx.gpu_id) as clk:
        for _ in range(steps):
            ctx.flush_l2()                                   # outside the step's events
            _, ev, spans = step(x, True)
            torch.cuda.synchronize()
            step_ms.append(ev[0][1].elapsed_time(ev[-1][1]))
            if spans:
                for n1, e0, e1 in spans:
                    kern_ms.setdefault(n1, []).append(e0.elapsed_time(e1))
            else:
                for (n0, e0), (n1, e1) in zip(ev[:-1], ev[1:]):
                    kern_ms.setdefault(n1, []).append(e0.elapsed_time(e1))
        torch.cuda.synchronize()
    ctx.barrier()
    mean_ms = max_over_ranks(sum(step_ms) / len(step_ms), dist, dev)

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if e2e_steps > 0:
        pinned = torch.from_numpy(host.view(np.int32) if as_words else host).pin_memory()
        e2e_ms = []
        d2h_bytes = 0
        for i in range(1 + e2e_steps):
            ctx.flush_l2()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            inp = pinned.to(dev, non_blocking=True)
            if as_words:
                inp = inp.view(torch.uint32)
            outs, _, _ = step(inp, False)
            host_outs = []
            for o in outs:
                h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
                h.copy_(o, non_blocking=True)
                host_outs.append(h)
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= 1:
                e2e_ms.append(e0.elapsed_time(e1))
            d2h_bytes = sum(o.numel() * o.element_size() for o in outs)
        e2e_mean = max_over_ranks(sum(e2e_ms) / len(e2e_ms), dist, dev)
    weak_units = rg is None
    units = w.n_seq * W.SEQ_LEN * (world if weak_units else 1)
    if e2e_steps > 0:
        e2e = {"value": units / (e2e_mean * 1e-3), "unit": "weights/s",
               "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": int(d2h_bytes),
               "steps": e2e_steps}

    # ---- near-ties of the Viterbi walks (an untimed call that also returns
    # each walk's smallest relative decision margin) ----
    near = None
    if "viterbi" in w.ops:
        _, _, mg = tcq.viterbi_encode(x, w.L, ws_v, D=Dd, margin=True)
        mg = mg.cpu().numpy()
        near = {"count": int((mg < NEAR_TIE).sum()), "threshold": NEAR_TIE, "sequences": int(mg.size),
                "min_margin": float(mg.min())}

    # ---- roofline of the dominant kernel ----
    from trellis_coded_weight_bitshift_b200 import roofline as RL
    kern_mean = {k: sum(v) / len(v) for k, v in kern_ms.items()}
    dom = max(kern_mean, key=kern_mean.get)
    peaks = RL.load_measured_peaks(ROOT)
    wl = W.Workload(**{**w.__dict__, "n_seq": n_local})
    roof = RL.roofline_entry(dom, wl, kern_mean[dom], peaks)
    clocks = clk.summary()
    rec = {
        "metric": _metric_for(w), "value": units / (mean_ms * 1e-3), "unit": "weights/s",
        "ms_per_step": mean_ms, "steps": steps, "warmup": warmup,
        "scaling": "weak" if weak_units else "strong",
        "kernels_ms": {k: round(v, 4) for k, v in kern_mean.items()},
        "edges_per_s": {k: RL.trellis_edges(k, wl) / (v * 1e-3) for k, v in kern_mean.items()
                        if RL.trellis_edges(k, wl) > 0},
        "roofline": roof, "gpu_launches": launches_per_step * steps,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
        "n_seq_per_gpu": n_local, "concurrent": concurrent,
    }
    if e2e is not None:
        rec["e2e"] = e2e
    if near is not None:
        rec["near_ties"] = near
    return rec


def run_ours(a) -> None:
    ctx = Ctx(a)
    w = W.WORKLOADS[a.workload]
    if a.n_seq and a.n_seq < w.n_seq:
        import dataclasses
        w = dataclasses.replace(w, n_seq=a.n_seq, rows=0, cols=0)
    # e2e repeats the step; a multi-second step repeats only a few times
    probe_long = w.name == DEFAULT_WORKLOAD and not a.n_seq
    e2e_steps = min(a.steps, 3) if probe_long else a.steps
    main = measure(ctx, w, a.steps, a.warmup, e2e_steps, a.weak)
    per = {}
    if not a.no_companions and a.workload == DEFAULT_WORKLOAD and not a.n_seq:
        for name in COMPANIONS:
            cw = W.WORKLOADS[name]
            rec = measure(ctx, cw, min(a.steps, 10), min(a.warmup, 3), 0, a.weak)
            per[name] = {k: rec[k] for k in ("metric", "value", "unit", "ms_per_step", "steps", "warmup",
                                             "scaling", "kernels_ms", "edges_per_s", "roofline",
                                             "gpu_launches", "clocks", "n_seq_per_gpu")}
            per[name]["roofline_frac"] = rec["roofline"]["frac"]
            if "near_ties" in rec:
                per[name]["near_ties"] = rec["near_ties"]
            per[name]["dtype"] = _dtype_for(cw)
    line = {
        "metric": main["metric"], "value": main["value"], "unit": "weights/s",
        "n_gpus": ctx.world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": main["ms_per_step"],
        "higher_is_better": True, "scaling": main["scaling"], "vs_baseline": None,
        "dtype": _dtype_for(w), "data": "synthetic",
        "config": {"workload": w.name, "L": w.L, "k": 2, "V": 1, "n_seq": w.n_seq,
                   "n_seq_per_gpu": main["n_seq_per_gpu"], "seq_len": W.SEQ_LEN, "temps": list(w.temps),
                   "ops": list(w.ops), "rows": w.rows, "cols": w.cols,
                   "l2": "flushed before every timed step, outside its events (256 MiB write, then "
                         "a 256 MiB read of another buffer, then a ~1 ms device spin)",
                   "parallelism": (f"dp{ctx.world}: " + ("each rank its own replica" if main["scaling"] == "weak"
                                   else "16x16-tile rows (or sequences) split across ranks")
                                   + ", no data-path collective"),
                   "streams": ("independent calls on separate streams (the batch under-fills the GPU)"
                               if main["concurrent"] else "one stream"),
                   "e2e_steps": e2e_steps},
        "kernels_ms": main["kernels_ms"], "edges_per_s": main["edges_per_s"],
        "roofline": main["roofline"], "gpu_launches": main["gpu_launches"], "clocks": main["clocks"],
    }
    if "e2e" in main:
        line["e2e"] = main["e2e"]
    if "near_ties" in main:
        line["near_ties"] = main["near_ties"]
    if per:
        line["per_workload"] = per
    if ctx.rank == 0 and ctx.world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if ctx.rank == 0:
        print(json.dumps(line))
    if ctx.dist is not None:
        ctx.dist.barrier()
        ctx.dist.destroy_process_group()


def main():
    a = _args()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
