"""nvfp4_global_scale_noalloc: the global scale for callers that cannot
allocate device memory (plugin hooks with no allocator, processes under a hard
memory cap).  It keeps its partial maxima in an array built into the library
instead of a caller workspace; its results must equal those of
nvfp4_global_scale, call after call, and the oracle's S.

This file is named to be collected last, so that a run stopping at the first
failure has run every other test before it.  It passes on its own in a fresh
process and after the rest of the suite."""
import ctypes as C

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _lib():
    import block_scale_search_b200 as nv
    L = nv.lib()
    f = L.nvfp4_global_scale_noalloc
    f.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_float, C.c_void_p, C.c_void_p,
                  C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    return nv, L


def _with_workspace(nv, W, q_max):
    S, amax, st = nv.global_scale(W, q_max)
    torch.cuda.synchronize()
    return S.item(), amax.item(), st.item()


def _no_alloc(L, W, q_max, S, amax, st):
    S.fill_(-1.0)
    amax.fill_(-1.0)
    st.fill_(99)
    rc = L.nvfp4_global_scale_noalloc(W.data_ptr(), W.shape[0], W.shape[1], W.stride(0),
                                      float(q_max), S.data_ptr(), amax.data_ptr(), st.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert rc == 0, rc
    torch.cuda.synchronize()
    return S.item(), amax.item(), st.item()


def test_no_alloc_global_scale_matches_workspace_version_twice():
    import oracle
    import workloads
    nv, L = _lib()
    S = torch.empty(1, device=DEV)
    amax = torch.empty(1, device=DEV)
    st = torch.empty(1, dtype=torch.int32, device=DEV)
    shapes = [(28672, 8192, 448.0, 31), (777, 1040, 256.0, 32)]   # two calls in a row
    Ws = [workloads.weight(o, i, 0.02, 0.001, 10.0, seed, DEV) for o, i, _, seed in shapes]
    refs = [_with_workspace(nv, W, q) for W, (_, _, q, _) in zip(Ws, shapes)]
    bad = workloads.weight(64, 64, 0.02, 0.0, 1.0, 33, DEV)
    bad[3, 5] = float("nan")
    _no_alloc(L, Ws[1], shapes[1][2], S, amax, st)  # first call on the device: its set-up
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated()
    free_before = torch.cuda.mem_get_info()[0]
    for W, (out, inp, q, _), ref in zip(Ws, shapes, refs):
        got = _no_alloc(L, W, q, S, amax, st)
        # the scale is exact: bit-equal to the workspace call ...
        assert np.float32(got[0]) == np.float32(ref[0]) and got[1] == ref[1] and got[2] == ref[2] == 0
        # ... and to the oracle's fl32(amax / fl32(Q * 6))
        S_ref, amax_ref, st_ref = oracle.global_scale(W.cpu().view(torch.uint16).numpy(), q)
        assert st_ref == 0 and np.float32(got[0]) == S_ref and np.float32(got[1]) == amax_ref
    # a matrix with a NaN reports it through the status word, like the original
    assert _no_alloc(L, bad, 448.0, S, amax, st)[2] == -5
    # nothing was allocated: neither through torch's caching allocator nor on
    # the device itself (free memory as the driver reports it)
    assert torch.cuda.memory_allocated() == torch_before
    assert torch.cuda.mem_get_info()[0] >= free_before


def test_no_alloc_rejects_bad_arguments_before_launch():
    _, L = _lib()
    P = 0x10000
    assert L.nvfp4_global_scale_noalloc(None, 4, 16, 16, 448.0, P, None, None, None) == -1
    assert L.nvfp4_global_scale_noalloc(P, 4, 12, 16, 448.0, P, None, None, None) == -2
    assert L.nvfp4_global_scale_noalloc(P + 2, 4, 16, 16, 448.0, P, None, None, None) == -3
    assert L.nvfp4_global_scale_noalloc(P, 4, 16, 16, 0.0, P, None, None, None) == -1
