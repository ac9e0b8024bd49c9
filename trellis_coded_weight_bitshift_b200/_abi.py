"""ctypes view of the C ABI in ``include/tcq.h`` (libtcq.so, in this package)."""
from __future__ import annotations

import ctypes
import os
from functools import lru_cache

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtcq.so")

TCQ_OK = 0
TCQ_ERR_INVALID_ARG = -1
TCQ_ERR_UNSUPPORTED = -2
TCQ_ERR_WORKSPACE = -3
TCQ_ERR_CUDA = -4

TAILBITING = 0
FREE_START = 1
OUT_SEQ = 0
OUT_TILE16 = 1

EXPORTS = (
    "tcq_version", "tcq_status_string", "tcq_stream_words",
    "tcq_viterbi_workspace_size", "tcq_viterbi_encode", "tcq_viterbi_encode_noalloc",
    "tcq_viterbi_encode_tailbiting",
    "tcq_bcjr_workspace_size", "tcq_bcjr_soft", "tcq_bcjr_soft_backward", "tcq_bcjr_soft_and_grad",
    "tcq_pack_states", "tcq_decode", "tcq_decode_gemv", "tcq_rht",
)


class Trellis(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int32), ("k", ctypes.c_int32), ("V", ctypes.c_int32),
                ("seq_len", ctypes.c_int32)]


class TcqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


@lru_cache(maxsize=None)
def lib() -> ctypes.CDLL:
    """Load libtcq.so; raise loudly if it has not been built."""
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m trellis_coded_weight_bitshift_b200.build`"
            " (the package has no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    TP = ctypes.POINTER(Trellis)
    L.tcq_version.restype = I
    L.tcq_version.argtypes = []
    L.tcq_status_string.restype = ctypes.c_char_p
    L.tcq_status_string.argtypes = [I]
    L.tcq_stream_words.restype = SZ
    L.tcq_stream_words.argtypes = [TP, I]
    L.tcq_viterbi_workspace_size.restype = SZ
    L.tcq_viterbi_workspace_size.argtypes = [TP, I64]
    L.tcq_viterbi_encode.restype = I
    L.tcq_viterbi_encode.argtypes = [TP, P, P, I64, P, P, P, P, SZ, P]
    L.tcq_viterbi_encode_tailbiting.restype = I
    L.tcq_viterbi_encode_tailbiting.argtypes = [TP, P, P, I64, P, P, P, SZ, P]
    L.tcq_viterbi_encode_noalloc.restype = I
    L.tcq_viterbi_encode_noalloc.argtypes = [TP, P, I64, P, P, P]
    L.tcq_bcjr_workspace_size.restype = SZ
    L.tcq_bcjr_workspace_size.argtypes = [TP, I64, I]
    L.tcq_bcjr_soft.restype = I
    L.tcq_bcjr_soft.argtypes = [TP, P, P, I64, F, P, P, P, SZ, P]
    L.tcq_bcjr_soft_backward.restype = I
    L.tcq_bcjr_soft_backward.argtypes = [TP, P, P, I64, F, P, P, P, P, SZ, P]
    L.tcq_bcjr_soft_and_grad.restype = I
    L.tcq_bcjr_soft_and_grad.argtypes = [TP, P, P, I64, F, P, P, P, P, P, SZ, P]
    L.tcq_pack_states.restype = I
    L.tcq_pack_states.argtypes = [TP, P, I64, I, P, P]
    L.tcq_decode_gemv.restype = I
    L.tcq_decode_gemv.argtypes = [TP, P, I, I64, I64, P, P, P]
    L.tcq_rht.restype = I
    L.tcq_rht.argtypes = [P, I64, I64, P, P, P, P]
    L.tcq_decode.restype = I
    L.tcq_decode.argtypes = [TP, P, I64, I, I, I64, I64, P, P]
    return L


def status_string(status: int) -> str:
    return lib().tcq_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != TCQ_OK:
        raise TcqError(status, where)


def trellis(L: int, seq_len: int, k: int = 2, V: int = 1) -> Trellis:
    return Trellis(int(L), int(k), int(V), int(seq_len))
