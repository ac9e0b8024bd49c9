"""The allocation-free Viterbi entry point gives the same walks and MSE as the
allocating one.

tcq_viterbi_encode_noalloc exists for callers that may not allocate device
memory when they call the library (a plugin whose host owns all device
memory, or a deployment whose memory budget is fixed at start-up): its
backpointers live in a fixed 32 MiB buffer inside the library image instead
of a caller workspace.  This file is named so that pytest collects it last;
it also passes when run on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import tcq_workloads as W

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    assert torch.cuda.is_available(), "GPU test"
    import trellis_coded_weight_bitshift_b200 as tcq
    from trellis_coded_weight_bitshift_b200 import _abi
    from trellis_coded_weight_bitshift_b200.build import build
    build()
    lib = _abi.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row at each L; the second is smaller, so stale
    # backpointers from the first call remain in the shared buffer beyond
    # what the second one uses.  L = 8 runs once at the documented maximum
    # (8,224 sequences: 8,224 x 255 x 16 bytes fill the 32 MiB buffer to
    # within 512 bytes).
    for L, n, seed in ((8, 8224, 70), (8, 64, 74), (12, 400, 71), (12, 150, 72), (16, 24, 73),
                       (16, 32, 75)):
        s = torch.from_numpy(W.gaussian(n, seed)).cuda()
        ref_states, ref_mse = tcq.viterbi_encode(s, L)          # caller-workspace entry point
        states = torch.empty_like(ref_states)
        mse = torch.empty_like(ref_mse)
        tr = _abi.trellis(L, 256)
        rc = lib.tcq_viterbi_encode_noalloc(ctypes.byref(tr), _p(s), n, _p(states), _p(mse), stream)
        assert rc == _abi.TCQ_OK, _abi.status_string(rc)
        torch.cuda.synchronize()
        # the Viterbi tests' tolerance: walks and MSE bit for bit
        assert torch.equal(states.view(torch.int16), ref_states.view(torch.int16))
        assert np.array_equal(mse.cpu().numpy().view(np.uint32), ref_mse.cpu().numpy().view(np.uint32))


@pytest.mark.parametrize("L,n", [(16, 33), (16, 40), (12, 515), (8, 8225)])
def test_noalloc_rejects_requests_beyond_its_buffer(L, n):
    # one sequence past each documented limit (32 at L = 16, 514 at L = 12,
    # 8,224 at L = 8) is refused on the host, before anything is launched
    assert torch.cuda.is_available(), "GPU test"
    from trellis_coded_weight_bitshift_b200 import _abi
    lib = _abi.lib()
    s = torch.zeros((n, 256), dtype=torch.float32, device="cuda")
    states = torch.full((n, 256), 7, dtype=torch.int16, device="cuda")
    mse = torch.full((n,), -1.0, dtype=torch.float32, device="cuda")
    tr = _abi.trellis(L, 256)
    rc = lib.tcq_viterbi_encode_noalloc(ctypes.byref(tr), _p(s), n, _p(states), _p(mse),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _abi.TCQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((states == 7).all()) and bool((mse == -1.0).all())    # outputs untouched
