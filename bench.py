"""Throughput of the bitshift-trellis hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of synthetic input:
for the default workload (L=12, 1024 x 256 i.i.d. N(0,1) weights) that is
Viterbi encode (forward + traceback, per-sequence MSE), packing the walks into
2-bit streams and decoding them back to fp16 weights, the BCJR soft codeword
at temp 0.05 and the gradient of the sum of soft codewords w.r.t. the targets
(soft codeword, log Z and gradient in one forward-backward sweep, since the
cotangent is known up front).
The metric is weights per second (whole job, all ranks).  Under torchrun each
rank encodes its own batch (weak scaling, no data-path collective); the step
time is the maximum over ranks of the CUDA-event time.

A batch that under-fills the GPU (the 64-sequence L=8 workload) runs its
independent calls (Viterbi and one soft pass per temperature) on separate
streams, each with its own workspace; every other workload runs on one stream.

Inputs (1 MiB) are smaller than L2, so L2 is flushed before every timed step,
outside the step's event pair: a 256 MiB write, then a 256 MiB read of another
buffer, which evicts the write's dirty lines so that the timed kernels do not
pay for writing them back; a ~1 ms device spin follows, so that the step's
launches are queued before the GPU reaches its first event.  `--impl reference` times the
plain CPU oracle on a bounded sample of the same workload (rank 0 only).
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

DEFAULT_WORKLOAD = "l12_gauss1024"



def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--n-seq", type=int, default=0,
                   help="encode only the first N sequences of the workload (profiling runs)")
    return p.parse_args()


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


def _weights_per_step(w: W.Workload) -> int:
    return w.n_seq * W.SEQ_LEN


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
def _oracle_step(w: W.Workload, s: np.ndarray, D=None) -> None:
    import oracle
    if "viterbi" in w.ops:
        st, _ = oracle.viterbi_f32(s, w.L, D=D)
        if "pack_decode" in w.ops:
            oracle.decode(oracle.pack(st, w.L, oracle.FREE_START), w.L, s.shape[1], oracle.FREE_START)
    if "viterbi_tb" in w.ops:
        oracle.viterbi_tailbiting_alg4_f32(s, w.L, D=D)
    for temp in w.temps:
        if "bcjr_grad" in w.ops and temp == w.temps[0]:
            oracle.bcjr_vjp(s, np.ones_like(s, dtype=np.float64), w.L, temp, D=D)  # also yields soft
        elif "bcjr" in w.ops:
            oracle.bcjr_soft(s, w.L, temp, D=D)


def _oracle_decode_step(bits: np.ndarray, w: W.Workload) -> None:
    import oracle
    if w.ops == ("gemv",):          # one band of tile-rows: decode, then the matvec
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


def cpu_baseline(w: W.Workload, budget_s: float = 12.0) -> dict:
    """Time the oracle, as it stands, on a bounded sample of the workload."""
    import oracle
    oracle.build()
    n_done, t0 = 0, time.perf_counter()
    if w.ops == ("rht",):
        done = 0
        while time.perf_counter() - t0 < 2.0:
            done += _oracle_rht_sample(w)
        dt = time.perf_counter() - t0
        return {"value": done / dt, "unit": "weights/s", "cores": os.cpu_count(), "kind": "oracle",
                "sample": f"dense-definition rotation of the leading {_RHT_SAMPLE[0]} x "
                          f"{_RHT_SAMPLE[1]} block of {w.name} (numpy matmul, all BLAS threads), "
                          f"{dt:.1f} s wall"}
    if w.ops in (("decode",), ("gemv",)):
        bits = W.streams(w.name)
        chunk = 1024
        while time.perf_counter() - t0 < budget_s and n_done + chunk <= bits.shape[0]:
            _oracle_decode_step(bits[n_done:n_done + chunk], w)
            n_done += chunk
    else:
        s = W.sequences(w.name, n_limit=min(w.n_seq, 256))
        D = W.weights(w.name, n_limit=min(w.n_seq, 256))
        while time.perf_counter() - t0 < budget_s and n_done < s.shape[0]:
            _oracle_step(w, s[n_done:n_done + 1], None if D is None else D[n_done:n_done + 1])
            n_done += 1
    dt = time.perf_counter() - t0
    return {"value": n_done * W.SEQ_LEN / dt, "unit": "weights/s", "cores": 1, "kind": "oracle",
            "sample": f"first {n_done} of {w.n_seq} sequences of {w.name}, single-threaded, "
                      f"{dt:.1f} s wall"}


def run_reference(a) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = W.WORKLOADS[a.workload]
    import oracle
    oracle.build()
    per_step = 1024 if w.ops in (("decode",), ("gemv",)) else 4   # sequences per bounded step
    wts = None
    if w.ops == ("rht",):
        times = []
        for i in range(a.warmup + a.steps):
            t0 = time.perf_counter()
            done = _oracle_rht_sample(w)
            if i >= a.warmup:
                times.append(time.perf_counter() - t0)
        step_s = sum(times) / len(times)
        value = done / step_s
        print(json.dumps({
            "impl": "reference", "metric": _metric_for(w), "value": value, "unit": "weights/s",
            "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "rows": w.rows, "cols": w.cols},
            "cpu_baseline": {"value": value, "unit": "weights/s", "cores": os.cpu_count(),
                             "kind": "oracle", "sample": "leading 256 x 1024 block per step"},
            "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return
    if w.ops in (("decode",), ("gemv",)):
        data = W.streams(w.name)[: per_step * (a.steps + a.warmup)]
    else:
        data = W.sequences(w.name, n_limit=min(w.n_seq, per_step * (a.steps + a.warmup)))
        wts = W.weights(w.name, n_limit=min(w.n_seq, per_step * (a.steps + a.warmup)))
    pos = 0
    times = []
    for i in range(a.warmup + a.steps):
        lo = pos % data.shape[0]
        chunk = data[lo: lo + per_step]
        pos += per_step
        t0 = time.perf_counter()
        if w.ops in (("decode",), ("gemv",)):
            _oracle_decode_step(chunk, w)
        else:
            _oracle_step(w, chunk, None if wts is None else wts[lo: lo + per_step])
        if i >= a.warmup:
            times.append(time.perf_counter() - t0)
    step_s = sum(times) / len(times)
    value = per_step * W.SEQ_LEN / step_s
    line = {
        "impl": "reference", "metric": _metric_for(w), "value": value, "unit": "weights/s",
        "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "L": w.L, "n_seq": w.n_seq,
                                        "seq_len": W.SEQ_LEN, "temps": list(w.temps)},
        "cpu_baseline": {"value": value, "unit": "weights/s", "cores": 1, "kind": "oracle",
                         "sample": f"{per_step} sequences per step of {w.name}, single-threaded"},
        "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ------------------------------------------------------------------ ranks
def rank_batch(w: W.Workload, rank: int) -> np.ndarray:
    """The batch rank `rank` encodes (weak scaling: every rank a batch of the
    workload's size, no data exchanged).  Rank 0 gets the workload itself;
    other ranks get draws of the same distribution from seed + 1000 * rank."""
    if w.ops == ("rht",):
        return W.student_t_block(w.seed + 1000 * rank, w.rows, w.cols)
    if w.ops in (("decode",), ("gemv",)):
        return W.bitstream(w.n_seq, w.seed + 1000 * rank)
    if rank == 0 or w.kind != "gaussian":
        return W.sequences(w.name, n_limit=w.n_seq)
    rng = np.random.default_rng(w.seed + 1000 * rank)
    return rng.standard_normal((w.n_seq, W.SEQ_LEN)).astype(np.float32)


def max_over_ranks(value: float, dist, device) -> float:
    """Step time of the job = the slowest rank's (a timing collective only)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ GPU arm
def run_ours(a) -> None:
    import torch
    import trellis_coded_weight_bitshift_b200 as tcq
    from trellis_coded_weight_bitshift_b200.build import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    if rank == 0:
        build()
    if dist is not None:
        dist.barrier()
    dev = torch.device("cuda", torch.cuda.current_device())
    w = W.WORKLOADS[a.workload]
    if a.n_seq and a.n_seq < w.n_seq:
        import dataclasses
        w = dataclasses.replace(w, n_seq=a.n_seq, rows=0, cols=0)

    # ---- inputs (each rank its own batch) ----
    host = rank_batch(w, rank)
    if w.ops in (("decode",), ("gemv",)):
        x = torch.from_numpy(host.view(np.int32)).to(dev).view(torch.uint32)
    else:
        x = torch.from_numpy(host).to(dev)
    h2d_bytes = host.nbytes
    if w.ops == ("gemv",):
        xvec = torch.from_numpy(W.gemv_vector(w.name)).to(dev)
        yvec = torch.empty((w.rows,), dtype=torch.float32, device=dev)
    if w.ops == ("rht",):
        _, s1h, s2h = W.rotation_input(w.name)
        sr, sc = torch.from_numpy(s1h).to(dev), torch.from_numpy(s2h).to(dev)
        rot_out = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.fill_(1)                                       # every line of L2 replaced ...
        flush_r.sum()                                        # ... and the dirty ones written back
        # keep the GPU busy for ~1 ms more, so that the step's first event and
        # launches are queued before the GPU reaches them: the events then time
        # the kernels, not the host's Python call overhead
        torch.cuda._sleep(2_000_000)

    ws_v = ws_b = ws_g = None
    if "viterbi" in w.ops or "viterbi_tb" in w.ops:
        ws_v = torch.empty(tcq.viterbi_workspace_size(w.L, 256, w.n_seq), dtype=torch.uint8, device=dev)
    if "bcjr" in w.ops and not ("bcjr_grad" in w.ops and len(w.temps) == 1):
        ws_b = torch.empty(tcq.bcjr_workspace_size(w.L, 256, w.n_seq), dtype=torch.uint8, device=dev)
    if "bcjr_grad" in w.ops:
        ws_g = torch.empty(tcq.bcjr_workspace_size(w.L, 256, w.n_seq, True), dtype=torch.uint8, device=dev)
    # a batch that under-fills the GPU runs its independent calls (Viterbi, one
    # soft pass per temperature) on separate streams, each with its own workspace
    concurrent = w.concurrent and "bcjr_grad" not in w.ops and "pack_decode" not in w.ops
    side = [torch.cuda.Stream(device=dev) for _ in range(1 + len(w.temps))] if concurrent else []
    ws_bt = ([torch.empty(tcq.bcjr_workspace_size(w.L, 256, w.n_seq), dtype=torch.uint8, device=dev)
              for _ in w.temps] if concurrent and "bcjr" in w.ops else [])
    ones = torch.ones((w.n_seq, W.SEQ_LEN), dtype=torch.float32, device=dev)
    wts = W.weights(w.name, n_limit=w.n_seq)
    Dd = torch.from_numpy(wts).to(dev) if wts is not None else None

    kern_ms: dict[str, list[float]] = {}
    launches_per_step = 0

    def step(inp, timed: bool):
        nonlocal launches_per_step
        outs = []
        ev = []
        spans = []                 # (name, start, end) of calls on side streams
        n_launch = 0

        def mark(name):
            if timed:
                e = torch.cuda.Event(enable_timing=True)
                e.record(stream)
                ev.append((name, e))

        if w.ops == ("gemv",):
            mark("start")
            out = tcq.decode_gemv(inp, xvec, w.rows, w.cols, L=w.L, out=yvec)
            mark("decode_gemv")
            n_launch += 1
            outs.append(out)
        elif w.ops == ("rht",):
            mark("start")
            out = tcq.rht(inp, sr, sc, out=rot_out)
            mark("rht")
            n_launch += 3
            outs.append(out)
        elif w.ops == ("decode",):
            mark("start")
            out = tcq.decode(inp, w.L, 256, tcq.TAILBITING, tcq.OUT_TILE16, w.rows, w.cols)
            mark("decode_tile16")
            n_launch += 1
            outs.append(out)
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

    for _ in range(a.warmup):
        step(x, False)
    torch.cuda.synchronize()

    # ---- device-timed region ----
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = []
    with ClockSampler(gpu_id) as clk:
        for _ in range(a.steps):
            flush_l2()                                       # outside the step's events
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
    if dist is not None:
        dist.barrier()
    mean_ms = max_over_ranks(sum(step_ms) / len(step_ms), dist, dev)

    # ---- end to end through the public API with host buffers ----
    as_words = w.ops in (("decode",), ("gemv",))
    pinned = torch.from_numpy(host.view(np.int32) if as_words else host).pin_memory()
    e2e_ms = []
    d2h_bytes = 0
    for i in range(a.warmup + a.steps):
        flush_l2()
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
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
        if i >= a.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
        d2h_bytes = sum(o.numel() * o.element_size() for o in outs)
    e2e_mean = max_over_ranks(sum(e2e_ms) / len(e2e_ms), dist, dev)

    units = _weights_per_step(w) * world
    clocks = clk.summary()

    # ---- roofline of the dominant kernel ----
    from trellis_coded_weight_bitshift_b200 import roofline as RL
    kern_mean = {k: sum(v) / len(v) for k, v in kern_ms.items()}
    dom = max(kern_mean, key=kern_mean.get)
    peaks = RL.load_measured_peaks(ROOT)
    roof = RL.roofline_entry(dom, w, kern_mean[dom], peaks)

    line = {
        "metric": _metric_for(w), "value": units / (mean_ms * 1e-3), "unit": "weights/s",
        "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": mean_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8" if w.ops == ("decode",) else "f32", "data": "synthetic",
        "config": {"workload": w.name, "L": w.L, "k": 2, "V": 1, "n_seq_per_gpu": w.n_seq,
                   "seq_len": W.SEQ_LEN, "temps": list(w.temps), "ops": list(w.ops),
                   "l2": "flushed before every timed step, outside its events (256 MiB write, then "
                         "a 256 MiB read of another buffer, then a ~1 ms device spin)",
                   "parallelism": f"dp{world} (independent batches, no data-path collective)",
                   "streams": ("independent calls on separate streams (the batch under-fills the GPU)"
                               if concurrent else "one stream")},
        "kernels_ms": {k: round(v, 4) for k, v in kern_mean.items()},
        "edges_per_s": {k: RL.trellis_edges(k, w) * world / (v * 1e-3) for k, v in kern_mean.items()
                        if RL.trellis_edges(k, w) > 0},
        "roofline": roof,
        "e2e": {"value": units / (e2e_mean * 1e-3), "unit": "weights/s",
                "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": int(d2h_bytes)},
        "gpu_launches": launches_per_step * a.steps,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    a = _args()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
