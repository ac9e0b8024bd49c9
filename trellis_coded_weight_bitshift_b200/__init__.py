"""Bitshift-trellis coded quantisation on NVIDIA B200 (sm_100a).

Thin PyTorch binding of ``libtcq.so`` (C ABI in ``include/tcq.h``).  Every
step of the computation runs in the library's CUDA kernels; this module only
checks tensor shapes, allocates outputs and workspaces with torch's caching
allocator and passes device pointers and the current CUDA stream.  There is
no CPU fallback: without the built library or a CUDA device every call raises.

Functions (QTIP blog "The trellis: a stateful codebook" / "The codebook is
computed" / "Tail-biting is worth its complexity"; BCJR-QAT abstract):
  viterbi_encode(s, L)                   -> (states uint16 [n,T], mse f32 [n])
  viterbi_encode_tailbiting(s, L)        -> tail-biting walks (2 bits per weight)
  bcjr_soft(s, L, temp)                  -> (soft f32 [n,T], log_z f32 [n])
  bcjr_soft_backward(s, L, temp, soft, g)-> grad_s f32 [n,T]
  bcjr_soft_and_grad(s, L, temp, g)      -> (soft, log_z, grad_s) in one sweep
  BcjrSoft.apply(s, L, temp)             -> soft (autograd through the VJP)
  pack_states(states, L, layout)         -> bits uint32 [n, words]
  decode(bits, L, T, layout, ...)        -> fp16 weights
  rht(W, sign_rows, sign_cols)           -> random-sign Hadamard rotation of W
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import (FREE_START, OUT_SEQ, OUT_TILE16, TAILBITING, TcqError, check, lib,
                   status_string, trellis)

__all__ = [
    "viterbi_encode", "viterbi_encode_tailbiting", "bcjr_soft", "bcjr_soft_and_grad", "bcjr_soft_backward", "BcjrSoft", "pack_states", "decode",
    "stream_words", "viterbi_workspace_size", "bcjr_workspace_size", "TcqError", "rht",
    "decode_gemv",
    "TAILBITING", "FREE_START", "OUT_SEQ", "OUT_TILE16", "lib", "status_string",
]


def _require_cuda(*tensors: "torch.Tensor | None") -> None:
    """Every tensor a call hands to the library (None entries skipped) is
    contiguous and on the current CUDA device, the one the library launches
    on: a host pointer, or another device's, would reach the kernels."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (no CPU fallback)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors must all be on one device ({dev} and {t.device})")
    if dev is not None and dev.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {dev} but the current device is "
                         f"cuda:{torch.cuda.current_device()} (select it with torch.cuda.device)")


def _out(out: torch.Tensor, shape, dtype, *like: torch.Tensor) -> torch.Tensor:
    """A caller's output tensor, checked before any launch: the kernels
    write all of ``shape`` in ``dtype`` through its pointer."""
    if tuple(out.shape) != tuple(shape) or out.dtype != dtype:
        raise ValueError(f"out must be a {dtype} tensor of shape {tuple(shape)}, "
                         f"not {out.dtype} {tuple(out.shape)}")
    _require_cuda(out, *like)
    return out


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: "torch.Tensor | None") -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _workspace(nbytes: int, device) -> torch.Tensor:
    # 256-byte aligned: the caching allocator hands out 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _use_workspace(workspace: "torch.Tensor | None", need: int, like: torch.Tensor) -> torch.Tensor:
    """The caller's workspace (any dtype, counted in bytes) when it holds
    ``need`` bytes, else a fresh one on ``like``'s device."""
    if workspace is not None:
        _require_cuda(workspace, like)
        if _nbytes(workspace) >= need:
            return workspace
    return _workspace(need, like.device)


def stream_words(L: int, seq_len: int, layout: int) -> int:
    return int(lib().tcq_stream_words(ctypes.byref(trellis(L, seq_len)), int(layout)))


def viterbi_workspace_size(L: int, seq_len: int, n_seq: int) -> int:
    return int(lib().tcq_viterbi_workspace_size(ctypes.byref(trellis(L, seq_len)), int(n_seq)))


def bcjr_workspace_size(L: int, seq_len: int, n_seq: int, with_grad: bool = False) -> int:
    return int(lib().tcq_bcjr_workspace_size(ctypes.byref(trellis(L, seq_len)), int(n_seq),
                                             int(bool(with_grad))))


def _weights(D: torch.Tensor | None, s: torch.Tensor) -> torch.Tensor | None:
    if D is None:
        return None
    _require_cuda(D, s)
    if D.shape != s.shape or D.dtype != torch.float32:
        raise ValueError("D must be a float32 tensor shaped like s")
    return D


def viterbi_encode(s: torch.Tensor, L: int, workspace: torch.Tensor | None = None,
                   D: torch.Tensor | None = None, margin: bool = False):
    """Min-MSE walk of every row of ``s`` [n, T] (fp32) on the (L, 2, 1)
    bitshift trellis with the 1MAD code; returns (states uint16, mse fp32),
    and with ``margin=True`` also the smallest relative decision margin along
    each walk (fp32 [n]; a second forward pass).  ``D`` (optional, same
    shape) weights each step's squared error."""
    _require_cuda(s)
    D = _weights(D, s)
    if s.dtype != torch.float32 or s.dim() != 2:
        raise ValueError("s must be a 2-D float32 tensor [n_seq, seq_len]")
    n, T = s.shape
    tr = trellis(L, T)
    states = torch.empty((n, T), dtype=torch.uint16, device=s.device)
    mse = torch.empty((n,), dtype=torch.float32, device=s.device)
    mrg = torch.empty((n,), dtype=torch.float32, device=s.device) if margin else None
    need = int(lib().tcq_viterbi_workspace_size(ctypes.byref(tr), n))
    ws = _use_workspace(workspace, need, s)
    check(lib().tcq_viterbi_encode(ctypes.byref(tr), _ptr(s), _ptr(D), n, _ptr(states), _ptr(mse),
                                   _ptr(mrg), _ptr(ws), _nbytes(ws), _stream()), "tcq_viterbi_encode")
    return (states, mse, mrg) if margin else (states, mse)


def viterbi_encode_tailbiting(s: torch.Tensor, L: int, workspace: torch.Tensor | None = None,
                              D: torch.Tensor | None = None):
    """Tail-biting walk of every row (two-run search: rotated free run, then a
    run with both ends pinned to the overlap read at the seam); returns
    (states uint16, mse fp32).  Pack the walk with layout TAILBITING."""
    _require_cuda(s)
    D = _weights(D, s)
    if s.dtype != torch.float32 or s.dim() != 2:
        raise ValueError("s must be a 2-D float32 tensor [n_seq, seq_len]")
    n, T = s.shape
    tr = trellis(L, T)
    states = torch.empty((n, T), dtype=torch.uint16, device=s.device)
    mse = torch.empty((n,), dtype=torch.float32, device=s.device)
    need = int(lib().tcq_viterbi_workspace_size(ctypes.byref(tr), n))
    ws = _use_workspace(workspace, need, s)
    check(lib().tcq_viterbi_encode_tailbiting(ctypes.byref(tr), _ptr(s), _ptr(D), n, _ptr(states),
                                              _ptr(mse), _ptr(ws), _nbytes(ws), _stream()),
          "tcq_viterbi_encode_tailbiting")
    return states, mse


def bcjr_soft(s: torch.Tensor, L: int, temp: float, workspace: torch.Tensor | None = None,
              D: torch.Tensor | None = None):
    """Soft codeword (Boltzmann expectation of the code at temperature
    ``temp``) of every row of ``s``; returns (soft fp32 [n,T], log_z fp32 [n])."""
    _require_cuda(s)
    D = _weights(D, s)
    if s.dtype != torch.float32 or s.dim() != 2:
        raise ValueError("s must be a 2-D float32 tensor [n_seq, seq_len]")
    n, T = s.shape
    tr = trellis(L, T)
    soft = torch.empty_like(s)
    logz = torch.empty((n,), dtype=torch.float32, device=s.device)
    need = int(lib().tcq_bcjr_workspace_size(ctypes.byref(tr), n, 0))
    ws = _use_workspace(workspace, need, s)
    check(lib().tcq_bcjr_soft(ctypes.byref(tr), _ptr(s), _ptr(D), n, float(temp), _ptr(soft),
                              _ptr(logz), _ptr(ws), _nbytes(ws), _stream()), "tcq_bcjr_soft")
    return soft, logz


def bcjr_soft_backward(s: torch.Tensor, L: int, temp: float, soft: torch.Tensor,
                       grad_soft: torch.Tensor, workspace: torch.Tensor | None = None,
                       D: torch.Tensor | None = None):
    """Vector-Jacobian product: grad_s[u] = sum_t grad_soft[t] d soft[t] / d s[u]."""
    _require_cuda(s, soft, grad_soft)
    D = _weights(D, s)
    if (s.dim() != 2 or s.shape != soft.shape or s.shape != grad_soft.shape
            or any(t.dtype != torch.float32 for t in (s, soft, grad_soft))):
        raise ValueError("s, soft and grad_soft must be float32 tensors of one shape [n_seq, seq_len]")
    n, T = s.shape
    tr = trellis(L, T)
    grad = torch.empty_like(s)
    need = int(lib().tcq_bcjr_workspace_size(ctypes.byref(tr), n, 1))
    ws = _use_workspace(workspace, need, s)
    check(lib().tcq_bcjr_soft_backward(ctypes.byref(tr), _ptr(s), _ptr(D), n, float(temp),
                                       _ptr(soft), _ptr(grad_soft), _ptr(grad), _ptr(ws),
                                       _nbytes(ws), _stream()), "tcq_bcjr_soft_backward")
    return grad


def bcjr_soft_and_grad(s: torch.Tensor, L: int, temp: float, grad_soft: torch.Tensor,
                       workspace: torch.Tensor | None = None, D: torch.Tensor | None = None):
    """Soft codeword, log Z and the vector-Jacobian product for a known
    cotangent ``grad_soft``, in one forward-backward sweep; returns
    (soft, log_z, grad_s)."""
    _require_cuda(s, grad_soft)
    D = _weights(D, s)
    if (s.dim() != 2 or s.shape != grad_soft.shape or s.dtype != torch.float32
            or grad_soft.dtype != torch.float32):
        raise ValueError("s and grad_soft must be float32 tensors of one shape [n_seq, seq_len]")
    n, T = s.shape
    tr = trellis(L, T)
    soft = torch.empty_like(s)
    logz = torch.empty((n,), dtype=torch.float32, device=s.device)
    grad = torch.empty_like(s)
    need = int(lib().tcq_bcjr_workspace_size(ctypes.byref(tr), n, 1))
    ws = _use_workspace(workspace, need, s)
    check(lib().tcq_bcjr_soft_and_grad(ctypes.byref(tr), _ptr(s), _ptr(D), n, float(temp),
                                       _ptr(grad_soft), _ptr(soft), _ptr(logz), _ptr(grad),
                                       _ptr(ws), _nbytes(ws), _stream()), "tcq_bcjr_soft_and_grad")
    return soft, logz, grad


class BcjrSoft(torch.autograd.Function):
    """soft = BcjrSoft.apply(s, L, temp[, D]): differentiable soft codeword."""

    @staticmethod
    def forward(ctx, s, L, temp, D=None):
        soft, _ = bcjr_soft(s, L, temp, D=D)
        ctx.save_for_backward(s, soft, D)
        ctx.L, ctx.temp = L, temp
        return soft

    @staticmethod
    def backward(ctx, g):
        s, soft, D = ctx.saved_tensors
        return bcjr_soft_backward(s, ctx.L, ctx.temp, soft, g.contiguous(), D=D), None, None, None


def pack_states(states: torch.Tensor, L: int, layout: int = FREE_START) -> torch.Tensor:
    """Pack walks [n, T] (uint16) into MSB-first bitstreams [n, words] (uint32)."""
    _require_cuda(states)
    if states.dtype != torch.uint16 or states.dim() != 2:
        raise ValueError("states must be a 2-D uint16 tensor")
    n, T = states.shape
    tr = trellis(L, T)
    words = int(lib().tcq_stream_words(ctypes.byref(tr), int(layout)))
    if words == 0:
        raise TcqError(_abi.TCQ_ERR_UNSUPPORTED, "tcq_stream_words")
    bits = torch.empty((n, words), dtype=torch.uint32, device=states.device)
    check(lib().tcq_pack_states(ctypes.byref(tr), _ptr(states), n, int(layout), _ptr(bits),
                                _stream()), "tcq_pack_states")
    return bits


def decode(bits: torch.Tensor, L: int, seq_len: int = 256, layout: int = TAILBITING,
           out_layout: int = OUT_SEQ, rows: int = 0, cols: int = 0,
           out: torch.Tensor | None = None) -> torch.Tensor:
    """Decode bitstreams [n, words] (uint32) into fp16 weights: [n, seq_len]
    (OUT_SEQ) or a [rows, cols] matrix of 16x16 tiles (OUT_TILE16)."""
    _require_cuda(bits)
    if bits.dtype != torch.uint32 or bits.dim() != 2:
        raise ValueError("bits must be a 2-D uint32 tensor")
    n = bits.shape[0]
    tr = trellis(L, seq_len)
    words = int(lib().tcq_stream_words(ctypes.byref(tr), int(layout)))
    if words == 0:
        raise TcqError(_abi.TCQ_ERR_UNSUPPORTED, "tcq_stream_words")
    if bits.shape[1] != words:
        raise ValueError(f"bits must have {words} words per sequence for this trellis and layout")
    shape = (rows, cols) if out_layout == OUT_TILE16 else (n, seq_len)
    if out is None:
        out = torch.empty(shape, dtype=torch.float16, device=bits.device)
    else:
        _out(out, shape, torch.float16, bits)
    check(lib().tcq_decode(ctypes.byref(tr), _ptr(bits), n, int(layout), int(out_layout), int(rows),
                           int(cols), _ptr(out), _stream()), "tcq_decode")
    return out


def rht(W: torch.Tensor, sign_rows: torch.Tensor, sign_cols: torch.Tensor,
        out: torch.Tensor | None = None) -> torch.Tensor:
    """Random-sign Hadamard rotation (H_R/sqrt R) diag(sign_rows) W
    diag(sign_cols) (H_C/sqrt C) of a fp32 matrix (``out`` may be ``W``)."""
    _require_cuda(W, sign_rows, sign_cols)
    if W.dim() != 2 or W.dtype != torch.float32:
        raise ValueError("W must be a 2-D float32 tensor")
    R, C = W.shape
    if sign_rows.shape != (R,) or sign_cols.shape != (C,):
        raise ValueError("sign vectors must match W's rows and columns")
    out = torch.empty_like(W) if out is None else _out(out, (R, C), torch.float32, W)
    check(lib().tcq_rht(_ptr(W), R, C, _ptr(sign_rows.float().contiguous()),
                        _ptr(sign_cols.float().contiguous()), _ptr(out), _stream()), "tcq_rht")
    return out


def decode_gemv(bits: torch.Tensor, x: torch.Tensor, rows: int, cols: int, L: int = 16,
                layout: int = TAILBITING, out: torch.Tensor | None = None) -> torch.Tensor:
    """y = W x with W the fp16 matrix decoded from 16x16-tile streams ``bits``,
    decoded in registers (never materialised); fp32 products and sums."""
    _require_cuda(bits, x)
    if bits.dtype != torch.uint32 or x.dtype != torch.float32 or x.shape != (cols,):
        raise ValueError("bits must be uint32 [tiles, words] and x float32 [cols]")
    tr = trellis(L, 256)
    words = int(lib().tcq_stream_words(ctypes.byref(tr), int(layout)))
    if bits.shape != ((rows // 16) * (cols // 16), words):
        raise ValueError("bits must hold one stream per 16x16 tile")
    y = (torch.empty((rows,), dtype=torch.float32, device=x.device) if out is None
         else _out(out, (rows,), torch.float32, x))
    check(lib().tcq_decode_gemv(ctypes.byref(tr), _ptr(bits), int(layout), int(rows), int(cols),
                                _ptr(x), _ptr(y), _stream()), "tcq_decode_gemv")
    return y
