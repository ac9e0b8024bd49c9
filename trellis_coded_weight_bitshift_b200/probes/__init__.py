"""Peak probes for the roofline denominators (run on the GPU).

    python -m trellis_coded_weight_bitshift_b200.probes

* pipe_peaks: per-SM results per clock of MUFU ex2/lg2, FFMA, FMNMX, packed
  FADD2 and compare+select (CUDA probe in pipe_peaks.cu, built with nvcc);
* write_peaks: write-only bandwidth of 1 GiB with this repository's own
  16-byte-store and bulk-copy kernels (CUDA probe in write_peaks.cu);
* stream_peaks: torch's byte fill and copy of 1 GiB buffers, best of 10 by
  CUDA events.  torch's uint8 fill is not a ceiling: 16-byte stores write
  about 1.6x faster on the same GPU.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))


def pipe_peaks() -> str:
    exe = os.path.join(ROOT, "_build", "pipe_peaks")
    os.makedirs(os.path.dirname(exe), exist_ok=True)
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe,
                           os.path.join(HERE, "pipe_peaks.cu")])
    return subprocess.run([exe], capture_output=True, text=True, check=True).stdout


def write_peaks() -> str:
    exe = os.path.join(ROOT, "_build", "write_peaks")
    os.makedirs(os.path.dirname(exe), exist_ok=True)
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe,
                           os.path.join(HERE, "write_peaks.cu")])
    return subprocess.run([exe], capture_output=True, text=True, check=True).stdout


def stream_peaks(nbytes: int = 1 << 30) -> str:
    import torch
    a = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    b = torch.empty_like(a)

    def best(f, reps=10):
        f()
        torch.cuda.synchronize()
        t = 1e30
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            t = min(t, e0.elapsed_time(e1))
        return t

    tw = best(lambda: a.fill_(7))
    tc = best(lambda: b.copy_(a))
    return (f"torch byte fill of {nbytes >> 20} MiB: {nbytes / tw / 1e6:.1f} GB/s\n"
            f"copy of {nbytes >> 20} MiB (read + write bytes): {2 * nbytes / tc / 1e6:.1f} GB/s\n")


if __name__ == "__main__":
    print(pipe_peaks())
    print(write_peaks())
    print(stream_peaks())
