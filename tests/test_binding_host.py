"""Host-side checks of the Python binding (no GPU needed).

The binding hands raw device pointers to ``libtcq.so``, which cannot see the
extent or the placement of a buffer.  So every tensor a call passes on must be
checked first: CPU tensors are refused (there is no CPU fallback), a caller's
output must have exactly the shape and dtype the kernels write, a caller's
workspace must be a device buffer, and a missing library must raise rather
than let anything run elsewhere.
"""
import os

import pytest
import torch

import trellis_coded_weight_bitshift_b200 as tcq
from trellis_coded_weight_bitshift_b200 import _abi


class _NoLaunch:
    """Stands in for the loaded library: the host-only size queries go to the
    real one, any other entry point fails the test."""

    HOST_ONLY = ("tcq_stream_words", "tcq_viterbi_workspace_size", "tcq_bcjr_workspace_size",
                 "tcq_status_string", "tcq_version")

    def __init__(self, real):
        self._real = real

    def __getattr__(self, name):
        if name in self.HOST_ONLY:
            return getattr(self._real, name)
        raise AssertionError(f"{name} was reached with host tensors")


@pytest.fixture
def no_launch(monkeypatch):
    from trellis_coded_weight_bitshift_b200.build import build
    build()
    real = _abi.lib()
    monkeypatch.setattr(tcq, "lib", lambda: _NoLaunch(real))


def test_every_entry_point_refuses_host_tensors(no_launch):
    s = torch.zeros(2, 256)
    D = torch.ones(2, 256)
    st = torch.zeros(2, 256, dtype=torch.int32).to(torch.uint16)
    bits = torch.zeros(4, 16, dtype=torch.int32).view(torch.uint32)
    W = torch.zeros(32, 32)
    sg = torch.ones(32)
    x = torch.zeros(32)
    calls = [
        lambda: tcq.viterbi_encode(s, 12),
        lambda: tcq.viterbi_encode(s, 12, D=D, margin=True),
        lambda: tcq.viterbi_encode_tailbiting(s, 12),
        lambda: tcq.bcjr_soft(s, 12, 1.0),
        lambda: tcq.bcjr_soft_backward(s, 12, 1.0, s, s),
        lambda: tcq.bcjr_soft_and_grad(s, 12, 1.0, s),
        lambda: tcq.BcjrSoft.apply(s, 12, 1.0),
        lambda: tcq.pack_states(st, 12, tcq.TAILBITING),
        lambda: tcq.decode(bits, 16, 256, tcq.TAILBITING, tcq.OUT_SEQ),
        lambda: tcq.decode(bits, 16, 256, tcq.TAILBITING, tcq.OUT_TILE16, 32, 32),
        lambda: tcq.rht(W, sg, sg),
        lambda: tcq.decode_gemv(bits, x, 32, 32),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()


def test_output_checks_come_before_the_device_check():
    # a caller's output is checked for the shape and dtype the kernels write
    # before anything else, so a wrong one is named even on the host
    for out, shape, dtype in ((torch.empty(31), (32,), torch.float32),
                              (torch.empty(32, dtype=torch.float16), (32,), torch.float32),
                              (torch.empty(32, 32), (32, 16), torch.float32),
                              (torch.empty(4, 256, dtype=torch.float16), (4, 255), torch.float16)):
        with pytest.raises(ValueError, match="out must be"):
            tcq._out(out, shape, dtype)
    with pytest.raises(ValueError, match="CUDA"):
        tcq._out(torch.empty(32), (32,), torch.float32)


def test_workspace_is_a_device_buffer_counted_in_bytes():
    with pytest.raises(ValueError, match="CUDA"):
        tcq._use_workspace(torch.empty(1 << 20, dtype=torch.uint8), 1024, torch.empty(2, 256))
    assert tcq._nbytes(torch.empty(10, dtype=torch.float32)) == 40
    assert tcq._nbytes(torch.empty(10, dtype=torch.uint8)) == 10
    assert tcq._nbytes(torch.empty(3, 5, dtype=torch.float16)) == 30


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "LIB_PATH", os.path.join(str(tmp_path), "libtcq.so"))
    _abi.lib.cache_clear()
    try:
        with pytest.raises(RuntimeError, match="no CPU fallback"):
            _abi.lib()
        with pytest.raises(RuntimeError, match="no CPU fallback"):
            tcq.stream_words(16, 256, tcq.TAILBITING)
    finally:
        monkeypatch.undo()
        _abi.lib.cache_clear()
    assert os.path.exists(_abi.LIB_PATH)
