"""Out-of-bounds writes: every C-ABI entry point, called on ragged sizes, writes
only inside its outputs and its workspace, and leaves its inputs unchanged.

Each output and workspace is carved from a larger device buffer whose bytes
before and after it (and the padding up to the next 256-byte boundary) hold a
sentinel pattern; after the call the sentinel must be intact.  This stands in
for a memory checker, which cannot be run on these GPUs.  Correctness of the
values is covered by the parity tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import tcq_workloads as W

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes of sentinel on each side (keeps 256-byte alignment)
FILL = 0xA5


@pytest.fixture(scope="module")
def abi():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from trellis_coded_weight_bitshift_b200 import _abi
    from trellis_coded_weight_bitshift_b200.build import build
    build()
    return _abi


class Guarded:
    """nbytes of device memory with sentinel bytes around it."""

    def __init__(self, nbytes: int):
        self.n = int(nbytes)
        body = (self.n + 255) // 256 * 256
        self.buf = torch.full((GUARD + body + GUARD,), FILL, dtype=torch.uint8, device="cuda")
        self.ptr = ctypes.c_void_p(self.buf.data_ptr() + GUARD)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.buf[:GUARD] == FILL).all()) and bool((self.buf[GUARD + self.n:] == FILL).all())


def _inp(a: np.ndarray):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t, t.clone(), ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _unchanged(*pairs):
    torch.cuda.synchronize()
    return all(torch.equal(a, b) for a, b in pairs)


@pytest.mark.parametrize("L,n,T", [(8, 5, 37), (8, 9, 256), (12, 5, 37), (12, 3, 256), (16, 3, 37)])
@pytest.mark.parametrize("weighted", [False, True])
def test_viterbi_writes_stay_inside(abi, L, n, T, weighted):
    lib = abi.lib()
    tr = abi.trellis(L, T)
    s, s0, sp = _inp(W.gaussian(n, 900 + T))
    D, D0, Dp = _inp(W.curvature(n, 901, seq_len=T)) if weighted else (s, s0, None)
    states, mse, margin = Guarded(n * T * 2), Guarded(n * 4), Guarded(n * 4)
    need = lib.tcq_viterbi_workspace_size(ctypes.byref(tr), n)
    ws = Guarded(need)
    rc = lib.tcq_viterbi_encode(ctypes.byref(tr), sp, Dp, n, states.ptr, mse.ptr, None, ws.ptr, need,
                                _stream())
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert states.intact() and mse.intact() and ws.intact()
    assert _unchanged((s, s0), (D, D0))
    # with the decision margins (a second forward pass that reads the walks)
    st0 = states.buf[GUARD:GUARD + n * T * 2].clone()
    rc = lib.tcq_viterbi_encode(ctypes.byref(tr), sp, Dp, n, states.ptr, mse.ptr, margin.ptr, ws.ptr,
                                need, _stream())
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert states.intact() and mse.intact() and margin.intact() and ws.intact()
    assert _unchanged((s, s0), (D, D0), (states.buf[GUARD:GUARD + n * T * 2], st0))


@pytest.mark.parametrize("L,n,T", [(8, 5, 48), (12, 3, 48), (16, 2, 256)])
def test_tailbiting_writes_stay_inside(abi, L, n, T):
    lib = abi.lib()
    tr = abi.trellis(L, T)
    s, s0, sp = _inp(W.gaussian(n, 910 + T))
    states, mse = Guarded(n * T * 2), Guarded(n * 4)
    need = lib.tcq_viterbi_workspace_size(ctypes.byref(tr), n)
    ws = Guarded(need)
    rc = lib.tcq_viterbi_encode_tailbiting(ctypes.byref(tr), sp, None, n, states.ptr, mse.ptr, ws.ptr,
                                           need, _stream())
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert states.intact() and mse.intact() and ws.intact()
    assert _unchanged((s, s0))


@pytest.mark.parametrize("L,n,T", [(8, 5, 37), (8, 11, 256), (12, 5, 37), (12, 2, 256), (16, 3, 37),
                                   (16, 2, 256)])
def test_bcjr_writes_stay_inside(abi, L, n, T):
    lib = abi.lib()
    tr = abi.trellis(L, T)
    temp = ctypes.c_float(0.2)
    s, s0, sp = _inp(W.gaussian(n, 920 + T))
    v, v0, vp = _inp(W.gaussian(n, 921 + T))
    st = _stream()
    # soft codeword and log Z
    soft, logz = Guarded(n * T * 4), Guarded(n * 4)
    need = lib.tcq_bcjr_workspace_size(ctypes.byref(tr), n, 0)
    ws = Guarded(need)
    rc = lib.tcq_bcjr_soft(ctypes.byref(tr), sp, None, n, temp, soft.ptr, logz.ptr, ws.ptr, need, st)
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert soft.intact() and logz.intact() and ws.intact()
    # separate backward, reading the soft codeword just written
    grad = Guarded(n * T * 4)
    needg = lib.tcq_bcjr_workspace_size(ctypes.byref(tr), n, 1)
    wsg = Guarded(needg)
    soft_t = soft.buf[GUARD:GUARD + n * T * 4].clone()
    rc = lib.tcq_bcjr_soft_backward(ctypes.byref(tr), sp, None, n, temp, soft.ptr, vp, grad.ptr,
                                    wsg.ptr, needg, st)
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert grad.intact() and wsg.intact()
    assert _unchanged((soft.buf[GUARD:GUARD + n * T * 4], soft_t))
    # one-sweep soft, log Z and gradient
    soft2, logz2, grad2 = Guarded(n * T * 4), Guarded(n * 4), Guarded(n * T * 4)
    wsg2 = Guarded(needg)
    rc = lib.tcq_bcjr_soft_and_grad(ctypes.byref(tr), sp, None, n, temp, vp, soft2.ptr, logz2.ptr,
                                    grad2.ptr, wsg2.ptr, needg, st)
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert soft2.intact() and logz2.intact() and grad2.intact() and wsg2.intact()
    assert _unchanged((s, s0), (v, v0))


@pytest.mark.parametrize("L", [8, 12, 16])
@pytest.mark.parametrize("T", [37, 256])
def test_pack_and_decode_writes_stay_inside(abi, L, T):
    lib = abi.lib()
    tr = abi.trellis(L, T)
    n = 7
    rng = np.random.default_rng(930 + L + T)
    st = np.empty((n, T), dtype=np.int64)
    st[:, 0] = rng.integers(0, 1 << L, n)
    for t in range(1, T):
        st[:, t] = ((st[:, t - 1] << 2) | rng.integers(0, 4, n)) & ((1 << L) - 1)
    states, states0, stp = _inp(st.astype(np.uint16).view(np.int16))
    for layout in (abi.TAILBITING, abi.FREE_START):
        if layout == abi.TAILBITING and (2 * T) % 32:
            continue
        words = lib.tcq_stream_words(ctypes.byref(tr), layout)
        bits = Guarded(n * words * 4)
        rc = lib.tcq_pack_states(ctypes.byref(tr), stp, n, layout, bits.ptr, _stream())
        assert rc == abi.TCQ_OK, abi.status_string(rc)
        assert bits.intact()
        out = Guarded(n * T * 2)
        rc = lib.tcq_decode(ctypes.byref(tr), bits.ptr, n, layout, abi.OUT_SEQ, 0, 0, out.ptr, _stream())
        assert rc == abi.TCQ_OK, abi.status_string(rc)
        assert out.intact()
    assert _unchanged((states, states0))


def test_decode_tiles_and_gemv_writes_stay_inside(abi):
    lib = abi.lib()
    tr = abi.trellis(16, 256)
    rows, cols = 48, 96
    n = (rows // 16) * (cols // 16)
    words = np.random.default_rng(940).integers(0, 2 ** 32, (n, 16), dtype=np.uint32)
    bits, bits0, bp = _inp(words.view(np.int32))
    out = Guarded(rows * cols * 2)
    rc = lib.tcq_decode(ctypes.byref(tr), bp, n, abi.TAILBITING, abi.OUT_TILE16, rows, cols, out.ptr,
                        _stream())
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert out.intact()
    x, x0, xp = _inp(W.gaussian(1, 941, seq_len=cols)[0])
    y = Guarded(rows * 4)
    rc = lib.tcq_decode_gemv(ctypes.byref(tr), bp, abi.TAILBITING, rows, cols, xp, y.ptr, _stream())
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert y.intact()
    assert _unchanged((bits, bits0), (x, x0))


@pytest.mark.parametrize("rows,cols", [(64, 128), (32, 8192), (1024, 32)])
def test_rht_writes_stay_inside(abi, rows, cols):
    lib = abi.lib()
    rng = np.random.default_rng(950 + rows)
    w, w0, wp = _inp(rng.standard_normal((rows, cols)).astype(np.float32))
    s1, s10, s1p = _inp((rng.integers(0, 2, rows) * 2 - 1).astype(np.float32))
    s2, s20, s2p = _inp((rng.integers(0, 2, cols) * 2 - 1).astype(np.float32))
    out = Guarded(rows * cols * 4)
    rc = lib.tcq_rht(wp, rows, cols, s1p, s2p, out.ptr, _stream())
    assert rc == abi.TCQ_OK, abi.status_string(rc)
    assert out.intact()
    assert _unchanged((w, w0), (s1, s10), (s2, s20))


def test_concurrent_streams_match_sequential(abi):
    # calls are re-entrant: the same calls on three streams at once (each with
    # its own workspace) give the same bits as one after another; the L = 16
    # kernels on two streams also exercise tensor-memory allocation on
    # shared SMs
    import trellis_coded_weight_bitshift_b200 as tcq
    s16 = torch.from_numpy(W.gaussian(300, 961)).cuda()
    s12 = torch.from_numpy(W.gaussian(1100, 962)).cuda()
    v12 = torch.from_numpy(W.gaussian(1100, 963)).cuda()

    def run():
        return (tcq.viterbi_encode(s16, 16), tcq.bcjr_soft(s16, 16, 0.3),
                tcq.bcjr_soft_and_grad(s12, 12, 0.1, v12))

    ref = run()
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(3)]
    cur = torch.cuda.current_stream()
    for st in streams:
        st.wait_stream(cur)
    with torch.cuda.stream(streams[0]):
        vit = tcq.viterbi_encode(s16, 16)
    with torch.cuda.stream(streams[1]):
        soft = tcq.bcjr_soft(s16, 16, 0.3)
    with torch.cuda.stream(streams[2]):
        sg = tcq.bcjr_soft_and_grad(s12, 12, 0.1, v12)
    torch.cuda.synchronize()
    got = (vit, soft, sg)
    for a, b in zip(got, ref):
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.int16) if x.dtype == torch.uint16 else x,
                               y.view(torch.int16) if y.dtype == torch.uint16 else y)


def test_binding_checks_callers_buffers_before_launch(abi):
    # The library sees only pointers, so the Python binding refuses, before
    # any launch, a caller's output that the kernels would write past (wrong
    # shape or dtype) or that is host memory, a host workspace, and
    # cotangents of the wrong dtype.  A caller's workspace of any dtype that
    # holds enough bytes is used and gives the same bits as an internal one.
    import trellis_coded_weight_bitshift_b200 as tcq
    bits = torch.zeros(4, 16, dtype=torch.int32, device="cuda").view(torch.uint32)
    for out in (torch.empty(4, 255, dtype=torch.float16, device="cuda"),
                torch.empty(4, 256, dtype=torch.float32, device="cuda"),
                torch.empty(4, 256, dtype=torch.float16)):
        with pytest.raises(ValueError, match="out must be|CUDA"):
            tcq.decode(bits, 16, 256, tcq.TAILBITING, tcq.OUT_SEQ, out=out)
    with pytest.raises(ValueError, match="out must be"):
        tcq.decode(bits, 16, 256, tcq.TAILBITING, tcq.OUT_TILE16, 32, 32,
                   out=torch.empty(32, 16, dtype=torch.float16, device="cuda"))
    wm = torch.zeros(16, 32, device="cuda")
    sr, sc = torch.ones(16, device="cuda"), torch.ones(32, device="cuda")
    for out in (torch.empty(32, 16, device="cuda"),
                torch.empty(16, 32, dtype=torch.float64, device="cuda"),
                torch.empty(16, 32)):
        with pytest.raises(ValueError, match="out must be|CUDA"):
            tcq.rht(wm, sr, sc, out=out)
    x = torch.zeros(32, device="cuda")
    for out in (torch.empty(31, device="cuda"),
                torch.empty(32, dtype=torch.float16, device="cuda"),
                torch.empty(32)):
        with pytest.raises(ValueError, match="out must be|CUDA"):
            tcq.decode_gemv(bits, x, 32, 32, out=out)

    s = torch.from_numpy(W.gaussian(3, 964)).cuda()
    with pytest.raises(ValueError, match="float32"):
        tcq.bcjr_soft_backward(s, 12, 1.0, s, s.half())
    with pytest.raises(ValueError, match="float32"):
        tcq.bcjr_soft_and_grad(s, 12, 1.0, s.double())
    with pytest.raises(ValueError, match="CUDA"):
        tcq.viterbi_encode(s, 12, workspace=torch.empty(1 << 20, dtype=torch.uint8))

    need_v = tcq.viterbi_workspace_size(12, 256, 3)
    need_b = tcq.bcjr_workspace_size(12, 256, 3)
    ws_v = torch.empty((need_v + 3) // 4, dtype=torch.float32, device="cuda")
    ws_b = torch.empty((need_b + 3) // 4, dtype=torch.float32, device="cuda")
    got = (tcq.viterbi_encode(s, 12, workspace=ws_v), tcq.bcjr_soft(s, 12, 0.5, workspace=ws_b))
    ref = (tcq.viterbi_encode(s, 12), tcq.bcjr_soft(s, 12, 0.5))
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        for u, v in zip(a, b):
            assert torch.equal(u.view(torch.int16) if u.dtype == torch.uint16 else u,
                               v.view(torch.int16) if v.dtype == torch.uint16 else v)
