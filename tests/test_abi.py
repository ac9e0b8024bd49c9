"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point that ``include/tcq.h`` declares, and rejects bad arguments
with the documented status codes before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_names():
    src = open(os.path.join(ROOT, "include", "tcq.h")).read()
    return sorted(set(re.findall(r"TCQ_API\s+[\w\s\*]+?\b(tcq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from trellis_coded_weight_bitshift_b200 import _abi
    from trellis_coded_weight_bitshift_b200.build import build
    build()
    return _abi.lib()


def test_header_declares_the_abi():
    names = _header_names()
    from trellis_coded_weight_bitshift_b200._abi import EXPORTS
    assert set(EXPORTS) == set(names), names


def test_library_exports_every_declared_symbol(L):
    for name in _header_names():
        assert hasattr(L, name), name


def test_status_strings(L):
    from trellis_coded_weight_bitshift_b200 import _abi
    for st in (0, -1, -2, -3, -4):
        assert len(_abi.status_string(st)) > 0
    assert L.tcq_version() >= 100


def test_invalid_arguments_return_status_without_launch(L):
    from trellis_coded_weight_bitshift_b200 import _abi
    tr = _abi.trellis(10, 256)                     # unsupported L
    bad = ctypes.c_void_p(16)                      # never dereferenced on these paths
    assert L.tcq_viterbi_encode(ctypes.byref(tr), bad, None, 1, bad, bad, None, bad, 1 << 20, None) == _abi.TCQ_ERR_UNSUPPORTED
    tr = _abi.trellis(12, 300)                     # seq_len above 256
    assert L.tcq_viterbi_encode(ctypes.byref(tr), bad, None, 1, bad, bad, None, bad, 1 << 20, None) == _abi.TCQ_ERR_UNSUPPORTED
    tr = _abi.trellis(12, 256, k=3)
    assert L.tcq_decode(ctypes.byref(tr), bad, 1, 0, 0, 0, 0, bad, None) == _abi.TCQ_ERR_UNSUPPORTED
    tr = _abi.trellis(12, 256)
    # null pointers
    assert L.tcq_viterbi_encode(ctypes.byref(tr), None, None, 4, bad, bad, None, bad, 1 << 20, None) == _abi.TCQ_ERR_INVALID_ARG
    # misaligned pointer
    assert L.tcq_viterbi_encode(ctypes.byref(tr), ctypes.c_void_p(18), None, 4, bad, bad, None, bad, 1 << 20, None) == _abi.TCQ_ERR_INVALID_ARG
    # workspace too small / missing / misaligned
    need = L.tcq_viterbi_workspace_size(ctypes.byref(tr), 4)
    assert need >= 4 * 255 * 256
    assert L.tcq_viterbi_encode(ctypes.byref(tr), bad, None, 4, bad, bad, None, ctypes.c_void_p(256), need - 1, None) == _abi.TCQ_ERR_WORKSPACE
    assert L.tcq_viterbi_encode(ctypes.byref(tr), bad, None, 4, bad, bad, None, None, need, None) == _abi.TCQ_ERR_WORKSPACE
    assert L.tcq_viterbi_encode(ctypes.byref(tr), bad, None, 4, bad, bad, None, ctypes.c_void_p(128), need, None) == _abi.TCQ_ERR_WORKSPACE
    # misaligned curvature weights
    assert L.tcq_viterbi_encode(ctypes.byref(tr), bad, ctypes.c_void_p(20), 4, bad, bad, None, bad, 1 << 20, None) == _abi.TCQ_ERR_INVALID_ARG
    # misaligned decision-margin output
    assert L.tcq_viterbi_encode(ctypes.byref(tr), bad, None, 4, bad, bad, ctypes.c_void_p(36), bad, 1 << 20, None) == _abi.TCQ_ERR_INVALID_ARG
    # nothing to do
    assert L.tcq_viterbi_encode(ctypes.byref(tr), None, None, 0, None, None, None, None, 0, None) == _abi.TCQ_OK
    # temperature must be positive and finite
    assert L.tcq_bcjr_soft(ctypes.byref(tr), bad, None, 4, ctypes.c_float(0.0), bad, None, bad, 1 << 30, None) == _abi.TCQ_ERR_INVALID_ARG
    assert L.tcq_bcjr_soft(ctypes.byref(tr), bad, None, 4, ctypes.c_float(float("inf")), bad, None, bad, 1 << 30, None) == _abi.TCQ_ERR_INVALID_ARG
    tr16 = _abi.trellis(16, 256)
    # the gradient entry points take L = 16 too; a missing workspace is caught on the host
    assert L.tcq_bcjr_soft_backward(ctypes.byref(tr16), bad, None, 4, ctypes.c_float(0.1), bad, bad, bad, None, 1 << 30, None) == _abi.TCQ_ERR_WORKSPACE
    assert L.tcq_bcjr_soft_and_grad(ctypes.byref(tr16), bad, None, 4, ctypes.c_float(0.1), bad, bad, None, bad, None, 1 << 30, None) == _abi.TCQ_ERR_WORKSPACE
    # decode: tile shape must cover exactly n_seq tiles
    assert L.tcq_decode(ctypes.byref(tr16), bad, 4, 0, 1, 32, 48, bad, None) == _abi.TCQ_ERR_INVALID_ARG
    assert L.tcq_decode(ctypes.byref(tr16), bad, 4, 0, 1, 32, 30, bad, None) == _abi.TCQ_ERR_INVALID_ARG
    assert L.tcq_decode(ctypes.byref(tr16), bad, 4, 7, 0, 0, 0, bad, None) == _abi.TCQ_ERR_INVALID_ARG


def test_stream_words(L):
    from trellis_coded_weight_bitshift_b200 import _abi
    for Lb in (8, 12, 16):
        tr = _abi.trellis(Lb, 256)
        assert L.tcq_stream_words(ctypes.byref(tr), _abi.TAILBITING) == 16
        assert L.tcq_stream_words(ctypes.byref(tr), _abi.FREE_START) == (512 + Lb - 2 + 31) // 32
    tr = _abi.trellis(16, 7)                       # 14 bits: too short to wrap a 16-bit window
    assert L.tcq_stream_words(ctypes.byref(tr), _abi.TAILBITING) == 0
    assert L.tcq_stream_words(ctypes.byref(tr), _abi.FREE_START) == 1


def test_empty_and_negative_batches_on_every_entry_point(L):
    # n_seq = 0 is an empty batch: TCQ_OK, nothing enqueued, no pointer read
    # (all are NULL here).  A negative count is an invalid argument.  Matrix
    # calls with a zero dimension are invalid (a 16x16 tile needs 16 of each).
    from trellis_coded_weight_bitshift_b200 import _abi
    f = ctypes.c_float
    for Lb in (8, 12, 16):
        tr = ctypes.byref(_abi.trellis(Lb, 256))
        calls = {
            "viterbi": lambda n: L.tcq_viterbi_encode(tr, None, None, n, None, None, None, None, 0, None),
            "noalloc": lambda n: L.tcq_viterbi_encode_noalloc(tr, None, n, None, None, None),
            "tailbiting": lambda n: L.tcq_viterbi_encode_tailbiting(tr, None, None, n, None, None, None, 0, None),
            "soft": lambda n: L.tcq_bcjr_soft(tr, None, None, n, f(0.1), None, None, None, 0, None),
            "backward": lambda n: L.tcq_bcjr_soft_backward(tr, None, None, n, f(0.1), None, None, None, None, 0,
                                                           None),
            "soft_and_grad": lambda n: L.tcq_bcjr_soft_and_grad(tr, None, None, n, f(0.1), None, None, None, None,
                                                                None, 0, None),
            "pack": lambda n: L.tcq_pack_states(tr, None, n, _abi.FREE_START, None, None),
            "decode": lambda n: L.tcq_decode(tr, None, n, _abi.TAILBITING, _abi.OUT_SEQ, 0, 0, None, None),
        }
        for name, call in calls.items():
            assert call(0) == _abi.TCQ_OK, (Lb, name)
            assert call(-1) == _abi.TCQ_ERR_INVALID_ARG, (Lb, name)
    tr16 = ctypes.byref(_abi.trellis(16, 256))
    assert L.tcq_decode_gemv(tr16, None, _abi.TAILBITING, 0, 16, None, None, None) == _abi.TCQ_ERR_INVALID_ARG
    assert L.tcq_decode_gemv(tr16, None, _abi.TAILBITING, 16, 0, None, None, None) == _abi.TCQ_ERR_INVALID_ARG
    assert L.tcq_rht(None, 0, 64, None, None, None, None) == _abi.TCQ_ERR_INVALID_ARG


def test_rht_arguments(L):
    # sizes: powers of two (else an invalid argument), 32 <= cols <= 8192 and
    # 32 <= rows <= 2^20 (else unsupported); every pointer non-null and
    # 16-byte aligned.  None of these calls reaches a launch.
    from trellis_coded_weight_bitshift_b200 import _abi
    p = ctypes.c_void_p(256)
    for rows, cols, want in ((48, 64, _abi.TCQ_ERR_INVALID_ARG), (64, 96, _abi.TCQ_ERR_INVALID_ARG),
                             (0, 64, _abi.TCQ_ERR_INVALID_ARG), (64, -64, _abi.TCQ_ERR_INVALID_ARG),
                             (16, 64, _abi.TCQ_ERR_UNSUPPORTED), (64, 16, _abi.TCQ_ERR_UNSUPPORTED),
                             (64, 16384, _abi.TCQ_ERR_UNSUPPORTED), (1 << 21, 64, _abi.TCQ_ERR_UNSUPPORTED)):
        assert L.tcq_rht(p, rows, cols, p, p, p, None) == want, (rows, cols)
    for i in range(4):                              # W, sign_rows, sign_cols, out
        for bad in (None, ctypes.c_void_p(256 + 4)):
            args = [p, p, p, p]
            args[i] = bad
            assert L.tcq_rht(args[0], 64, 64, args[1], args[2], args[3], None) == _abi.TCQ_ERR_INVALID_ARG, (i, bad)
