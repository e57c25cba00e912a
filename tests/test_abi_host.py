"""The C ABI without a GPU: the library loads, exports every function that
include/*.h declares, and rejects bad arguments on the host (before any CUDA
call) with the documented status codes."""
import ctypes as C
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session")
def L():
    from block_scale_search_b200 import _build, lib
    _build.build()
    return lib()


def declared_functions():
    names = []
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b(nvfp4_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert "nvfp4_scale_sweep_quantize" in names and len(names) >= 8
    out = subprocess.run(["nm", "-D", "--defined-only", L._name], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (nvfp4_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L, n)


def test_version(L):
    assert L.nvfp4_version() == 100


P = 0x10000  # a 64 KiB-aligned fake device address: never dereferenced (checks fail first)


def test_diag_hessian_validation(L):
    f = L.nvfp4_diag_hessian
    ws = P
    assert f(None, 4, 16, 16, P, 0, ws, 1 << 20, None) == -1          # X NULL with tokens
    assert f(P, 4, 16, 16, None, 0, ws, 1 << 20, None) == -1          # h NULL
    assert f(P, -1, 16, 16, P, 0, ws, 1 << 20, None) == -1            # negative tokens
    assert f(P, 4, 16, 16, P, 2, ws, 1 << 20, None) == -1             # accumulate flag
    assert f(P, 4, 12, 16, P, 0, ws, 1 << 20, None) == -2             # in % 8
    assert f(P, 4, 16, 8, P, 0, ws, 1 << 20, None) == -2              # ldx < in
    assert f(P + 2, 4, 16, 16, P, 0, ws, 1 << 20, None) == -3         # X misaligned
    assert f(P, 4, 16, 20, P, 0, ws, 1 << 20, None) == -3             # ldx % 8
    assert f(P, 4, 16, 16, P + 2, 0, ws, 1 << 20, None) == -3         # h misaligned
    assert f(P, 4, 16, 16, P, 0, None, 1 << 20, None) == -7           # no workspace
    assert f(P, 4, 16, 16, P, 0, ws + 4, 1 << 20, None) == -3         # workspace misaligned


def test_global_scale_validation(L):
    f = L.nvfp4_global_scale
    assert f(None, 4, 16, 16, 448.0, P, None, None, P, 1024, None) == -1
    assert f(P, 4, 16, 16, 448.0, None, None, None, P, 1024, None) == -1   # S NULL
    assert f(P, 4, 16, 16, 0.0, P, None, None, P, 1024, None) == -1       # q_max <= 0
    assert f(P, 4, 16, 16, float("inf"), P, None, None, P, 1024, None) == -1
    assert f(P, 4, 12, 16, 448.0, P, None, None, P, 1024, None) == -2      # in % 8
    assert f(P, 4, 16, 8, 448.0, P, None, None, P, 1024, None) == -2       # ldw < in
    assert f(P + 8, 4, 16, 16, 448.0, P, None, None, P, 1024, None) == -3  # W misaligned
    assert f(P, 4, 16, 16, 448.0, P + 1, None, None, P, 1024, None) == -3  # S misaligned
    assert f(P, 4, 16, 16, 448.0, P, None, None, None, 1024, None) == -7   # no workspace


def test_sweep_validation(L):
    f = L.nvfp4_scale_sweep_quantize
    ok = (P, 4, 32, 32, None, P, -9, 6, P, P, None, None)

    def call(**kw):
        names = ["W", "out", "inp", "ldw", "h", "S", "lo", "hi", "codes", "scales", "offs", "st"]
        a = dict(zip(names, ok))
        a.update(kw)
        return f(*[a[n] for n in names])

    assert call(W=None) == -1
    assert call(S=None) == -1
    assert call(codes=None) == -1
    assert call(scales=None) == -1
    assert call(out=-1) == -1
    assert call(inp=24, ldw=24) == -2                 # in % 16
    assert call(ldw=16) == -2                         # ldw < in
    assert call(W=P + 4) == -3
    assert call(ldw=36) == -3                         # ldw % 8
    assert call(h=P + 4) == -3                        # h must be 16-byte aligned
    assert call(codes=P + 4) == -3
    for lo, hi in ((1, 6), (-9, -1), (-17, 0), (0, 16), (-9, 7), (-16, 1)):
        assert call(lo=lo, hi=hi) == -4, (lo, hi)
    assert call(out=0) == 0                           # empty: nothing to do, no device needed
    assert call(inp=0, ldw=0) == 0


def test_dequantize_validation(L):
    f = L.nvfp4_dequantize
    assert f(P, P, P, -1, 16, P, None) == -1
    assert f(P, P, P, 2, 24, P, None) == -2
    assert f(None, P, P, 2, 16, P, None) == -1
    assert f(P + 4, P, P, 2, 16, P, None) == -3
    assert f(P, P, P, 2, 16, P + 8, None) == -3
    assert f(P, P, P, 0, 16, P, None) == 0


def test_binding_has_same_names_as_abi():
    import block_scale_search_b200 as m
    for n in declared_functions():
        if n == "nvfp4_last_cuda_error":
            continue
        assert hasattr(m, n), n


def test_grouped_and_batched_validation(L):
    import block_scale_search_b200 as nv
    f = L.nvfp4_diag_hessian_grouped
    f.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_int64, C.c_void_p,
                  C.c_int, C.c_void_p, C.c_size_t, C.c_void_p]
    ws = 0x100000
    assert f(P, None, 4, 100, 64, 64, P, 0, ws, 1 << 30, None) == -1        # no offsets
    assert f(P, P, 0, 100, 64, 64, P, 0, ws, 1 << 30, None) == -1           # no experts
    assert f(P, P, 70000, 100, 64, 64, P, 0, ws, 1 << 30, None) == -2       # too many experts
    assert f(P, P + 4, 4, 100, 64, 64, P, 0, ws, 1 << 30, None) == -3       # offsets misaligned
    assert f(P, P, 4, 100, 64, 64, P, 0, ws + 16, 1 << 30, None) == -3      # workspace alignment
    assert f(P, P, 4, 100, 64, 64, P, 0, ws, 16, None) == -7                # workspace too small
    assert L.nvfp4_diag_hessian_grouped_workspace_size(0, 4, 64) == 0 or \
        L.nvfp4_diag_hessian_grouped_workspace_size(100, 4, 64) >= 5 * 64 * 4  # device-dependent

    g = L.nvfp4_global_scale_batched
    good = [nv.MatrixDesc(P, 4, 16, 16), nv.MatrixDesc(P, 2, 32, 40)]
    arr = (nv.MatrixDesc * 2)(*good)
    bad = (nv.MatrixDesc * 2)(nv.MatrixDesc(P, 4, 16, 16), nv.MatrixDesc(P + 2, 2, 32, 40))
    assert g(bad, 2, 448.0, P, None, None, ws, 1 << 20, None) == -3
    bad = (nv.MatrixDesc * 1)(nv.MatrixDesc(P, 4, 12, 16))
    assert g(bad, 1, 448.0, P, None, None, ws, 1 << 20, None) == -2
    assert g(None, 3, 448.0, P, None, None, ws, 1 << 20, None) == -1
    assert g(arr, 2, 0.0, P, None, None, ws, 1 << 20, None) == -1
    assert g(arr, 0, 448.0, P, None, None, None, 0, None) == 0             # empty batch

    s = L.nvfp4_scale_sweep_quantize_batched
    d = [nv.SweepDesc(P, 4, 32, 32, P, P, P, P, None), nv.SweepDesc(P, 4, 32, 32, None, P, P, P, None)]
    arr = (nv.SweepDesc * 2)(*d)
    assert s(arr, 2, -9, 6, ws, 1 << 20, None) == -1                        # mixed objectives
    arr1 = (nv.SweepDesc * 1)(d[0])
    assert s(arr1, 1, -9, 7, ws, 1 << 20, None) == -4                       # window too wide
    arr1 = (nv.SweepDesc * 1)(nv.SweepDesc(P, 4, 24, 32, None, P, P, P, None))
    assert s(arr1, 1, -9, 6, ws, 1 << 20, None) == -2                       # in % 16
    arr1 = (nv.SweepDesc * 1)(nv.SweepDesc(P, 4, 32, 32, P + 4, P, P, P, None))
    assert s(arr1, 1, -9, 6, ws, 1 << 20, None) == -3                       # h alignment
    arr1 = (nv.SweepDesc * 1)(d[1])
    assert s(arr1, 1, -9, 6, None, 0, None) == -7                           # no workspace
    assert s(None, 0, -9, 6, None, 0, None) == 0                            # empty batch


def test_activation_validation(L):
    f = L.nvfp4_quantize_activations
    names = ["A", "tokens", "inp", "lda", "q", "lo", "hi", "S", "codes", "scales", "offs", "st",
             "stream"]
    ok = (P, 4, 32, 32, 256.0, -3, 7, P, P, P, None, None, None)

    def call(**kw):
        a = dict(zip(names, ok))
        a.update(kw)
        return f(*[a[n] for n in names])

    assert call(A=None) == -1
    assert call(S=None) == -1
    assert call(codes=None) == -1
    assert call(scales=None) == -1
    assert call(tokens=-1) == -1
    assert call(q=0.0) == -1
    assert call(q=float("nan")) == -1
    assert call(inp=24, lda=24) == -2                 # in % 16
    assert call(lda=16) == -2                         # lda < in
    assert call(A=P + 8) == -3
    assert call(lda=36) == -3                         # lda % 8
    assert call(S=P + 2) == -3
    assert call(codes=P + 4) == -3
    assert call(st=P + 2) == -3
    for lo, hi in ((1, 6), (-3, -1), (-17, 0), (0, 16), (-9, 7)):
        assert call(lo=lo, hi=hi) == -4, (lo, hi)
    assert call(tokens=0, S=None, codes=None, scales=None) == 0   # empty, no status: no device


def test_blocked_scales_validation(L):
    f = L.nvfp4_scales_to_blocked
    assert L.nvfp4_blocked_scales_size(300, 130) == 384 * 132
    assert L.nvfp4_blocked_scales_size(128, 4) == 512
    assert L.nvfp4_blocked_scales_size(-1, 4) == 0
    assert f(P, -1, 4, 4, P, None) == -1
    assert f(P, 4, 8, 4, P, None) == -2              # ld < cols
    assert f(None, 4, 4, 4, P, None) == -1
    assert f(P, 4, 4, 4, None, None) == -1
    assert f(P, 4, 4, 4, P + 8, None) == -3          # out must be 16-byte aligned
    assert f(P, 0, 4, 4, None, None) == 0            # empty


def test_debug_row_counters_validation(L):
    p, n = C.c_void_p(), C.c_size_t()
    assert L.nvfp4_debug_row_counters(None, C.byref(n)) == -1
    assert L.nvfp4_debug_row_counters(C.byref(p), None) == -1
    import torch
    if not torch.cuda.is_available():   # no device: a CUDA error, not a crash
        assert L.nvfp4_debug_row_counters(C.byref(p), C.byref(n)) == -6


def test_quantize_layer_validation(L):
    import block_scale_search_b200 as nv
    W = lambda **k: nv.LayerWeight(**{**dict(W=P, out=64, inp=256, ldw=256, input=0, S=P, amax=None,
                                            status=None, codes=P, scales=P, chosen_offset=None), **k})
    X = lambda **k: nv.LayerInput(**{**dict(X=P, tokens=32, inp=256, ldx=256, h=P), **k})
    ws = P

    def call(ws_list, xs_list, q=448.0, lo=-9, hi=6, nb=1 << 30):
        wa = (nv.LayerWeight * max(1, len(ws_list)))(*ws_list)
        xa = (nv.LayerInput * max(1, len(xs_list)))(*xs_list)
        return L.nvfp4_quantize_layer(wa, len(ws_list), xa, len(xs_list), q, lo, hi, ws, nb, None, None)

    assert call([W(input=1)], [X()]) == -1                 # input index out of range
    assert call([W(input=-2)], [X()]) == -1
    assert call([W(S=None)], [X()]) == -1                  # S missing
    assert call([W(inp=128, ldw=128)], [X()]) == -2        # in differs from the input's
    assert call([W(out=0)], [X()]) == -2                   # empty weight
    assert call([W(inp=72, ldw=72)], [X(inp=72, ldx=72)]) == -2   # in % 16
    assert call([W(W=P + 8)], [X()]) == -3                 # W misaligned
    assert call([W()], [X(h=P + 4)]) == -3                 # h not 16-byte aligned
    assert call([W()], [X(tokens=-1)]) == -1
    assert call([W()], [X()], q=float("nan")) == -1
    assert call([W()], [X()], lo=-10, hi=6) == -4          # window over 16
    assert L.nvfp4_quantize_layer(None, 1, None, 0, 448.0, -9, 6, ws, 1 << 30, None, None) == -1
    # the order query validates as the call does
    order = (C.c_int * 1)()
    wa1 = (nv.LayerWeight * 1)(W())
    xa1 = (nv.LayerInput * 1)(X())
    assert L.nvfp4_quantize_layer_order(wa1, 1, xa1, 1, -10, 6, order) == -4
    assert L.nvfp4_quantize_layer_order(wa1, 1, xa1, 1, -9, 6, None) == -1
    wbad = (nv.LayerWeight * 1)(W(input=1))
    assert L.nvfp4_quantize_layer_order(wbad, 1, xa1, 1, -9, 6, order) == -1
    # no device here: the workspace query returns 0 and a valid call a CUDA error
    import torch
    if not torch.cuda.is_available():
        wa = (nv.LayerWeight * 1)(W())
        xa = (nv.LayerInput * 1)(X())
        assert L.nvfp4_quantize_layer_workspace_size(wa, 1, xa, 1) == 0
        assert call([W()], [X()]) == -6
        assert L.nvfp4_quantize_layer_order(wa, 1, xa, 1, -9, 6, order) == -6


def test_quantize_layers_validation(L):
    """The multi-layer call checks each layer's descriptors as the one-layer
    call does, with input indices local to their layer."""
    import block_scale_search_b200 as nv
    W = lambda **k: nv.LayerWeight(**{**dict(W=P, out=64, inp=256, ldw=256, input=0, S=P, amax=None,
                                            status=None, codes=P, scales=P, chosen_offset=None), **k})
    X = lambda **k: nv.LayerInput(**{**dict(X=P, tokens=32, inp=256, ldx=256, h=P), **k})

    def call(layers, n=None, q=448.0, lo=-9, hi=6):
        arr, _keep = nv._layers_array(layers)
        return L.nvfp4_quantize_layers(arr, len(layers) if n is None else n, q, lo, hi, P, 1 << 30,
                                       None, None)

    assert L.nvfp4_quantize_layers(None, 1, 448.0, -9, 6, P, 1 << 30, None, None) == -1
    assert call([([W()], [X()])], n=-1) == -1
    # layer 1's weight names its own input 1, which layer 1 does not have
    assert call([([W()], [X()]), ([W(input=1)], [X()])]) == -1
    assert call([([W()], [X()]), ([W(input=0, inp=128, ldw=128)], [X()])]) == -2
    assert call([([W()], [X()]), ([W()], [X(h=P + 4)])]) == -3
    assert call([([W()], [X()])], lo=-10) == -4
    assert call([]) == 0                                    # nothing to do
    import torch
    if not torch.cuda.is_available():
        arr, _keep = nv._layers_array([([W()], [X()]), ([W(), W(input=-1)], [X()])])
        assert L.nvfp4_quantize_layers_workspace_size(arr, 2) == 0
        assert call([([W()], [X()]), ([W(), W(input=-1)], [X()])]) == -6


def test_grouped_layer_order(L):
    """The grouped layer call sweeps first the batch whose order costs less:
    with the 128-expert layer's sizes, the down projections (whose input is
    the smaller) go first and the gate/up input's h is streamed beside their
    sweep; passed the other way round, the caller's order stands.  A batch
    whose h point into the other input's h never goes first.  Host only."""
    import block_scale_search_b200 as nv
    E, T = 128, 2_097_152
    h1, h2 = 0x100000, 0x200000          # the two inputs' h [E, in]
    S = 0x300000
    x_gu = nv.GroupedInput(P, P, T, 2048, 2048, h1)
    x_dn = nv.GroupedInput(P, P, T, 768, 768, h2)

    def descs(shape, n, hbase, in_, s0):
        return [nv.SweepDesc(P, shape[0], shape[1], shape[1], hbase + 4 * in_ * (i % E),
                             S + 4 * (s0 + i), P, P, None) for i in range(n)]

    gu = descs((768, 2048), 2 * E, h1, 2048, 0)
    dn = descs((2048, 768), E, h2, 768, 2 * E)
    assert nv.nvfp4_quantize_grouped_layer_order(gu, dn, x_gu, x_dn, E, S, -9, 6) == 1
    # the other way round: the down batch is already first
    dn0 = descs((2048, 768), E, h2, 768, 0)
    gu1 = descs((768, 2048), 2 * E, h1, 2048, E)
    assert nv.nvfp4_quantize_grouped_layer_order(dn0, gu1, x_dn, x_gu, E, S, -9, 6) == 0
    # the second batch reading the first input's h cannot go first
    dn_bad = descs((2048, 768), E, h1, 2048, 2 * E)
    assert nv.nvfp4_quantize_grouped_layer_order(gu, dn_bad, x_gu, x_dn, E, S, -9, 6) == 0
    # a small first input and a large sweep keep the caller's order even when
    # the second input is larger: its reduction is carried at a fraction of its cost
    x_small = nv.GroupedInput(P, P, 4096, 2048, 2048, h1)
    x_big = nv.GroupedInput(P, P, 65536, 768, 768, h2)
    assert nv.nvfp4_quantize_grouped_layer_order(gu, dn, x_small, x_big, E, S, -9, 6) == 0
    # an empty first batch cannot carry anything: the second goes first
    assert nv.nvfp4_quantize_grouped_layer_order([], descs((2048, 768), E, h2, 768, 0), x_gu, x_dn,
                                                 E, S, -9, 6) == 1
    # invalid arguments: the validation's status
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_quantize_grouped_layer_order(gu, dn, x_gu, x_dn, E, S, -10, 6)
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_quantize_grouped_layer_order(gu, dn, x_gu, x_dn, E, S + 4, -9, 6)


def test_every_launching_entry_point_opens_an_nvtx_range():
    """Each entry point that enqueues GPU work opens a named NVTX range first
    (a profiler timeline then shows which call launched which kernels); the
    size and order queries, which launch nothing, need none."""
    import re
    csrc = os.path.join(ROOT, "block_scale_search_b200", "csrc")
    found = {}
    for fn in ("nvfp4hs_capi.cu", "global_scale_noalloc.cu"):
        src = open(os.path.join(csrc, fn)).read()
        for m in re.finditer(r"\n(?:extern \"C\" )?int (nvfp4_\w+)\((?:.|\n)*?\) \{\n(.*)\n", src):
            found[m.group(1)] = m.group(2).strip()
    queries = {"nvfp4_version", "nvfp4_last_cuda_error", "nvfp4_quantize_layer_order",
               "nvfp4_debug_checks_compiled", "nvfp4_debug_checks",
               "nvfp4_quantize_grouped_layer_order", "nvfp4_debug_row_counters",
               "nvfp4_gptq_set_timing", "nvfp4_gptq_phase_times"}
    launching = {k: v for k, v in found.items() if k not in queries}
    assert len(launching) == 16, sorted(launching)
    for name, first in launching.items():
        assert first == f'NVFP4_RANGE("{name}");', (name, first)


def test_checked_build_loads_and_exports_the_same_entry_points():
    """The bounds-checked variant is built beside the library (CPU compile),
    exports every entry point the header declares, and says which it is."""
    import ctypes as C
    from block_scale_search_b200 import _build
    path = _build.build(checked=True)
    Lc = C.CDLL(path)
    Lp = C.CDLL(_build.LIB)
    for name in declared_functions():
        assert hasattr(Lc, name), name
    assert Lc.nvfp4_debug_checks_compiled() == 1 and Lp.nvfp4_debug_checks_compiled() == 0
    first, count = C.c_ulonglong(7), C.c_uint(7)
    assert Lp.nvfp4_debug_checks(C.byref(first), C.byref(count), 0) == 0
    assert first.value == 0 and count.value == 0            # nothing recorded without checks
    assert Lp.nvfp4_debug_checks(None, C.byref(count), 0) == -1


def test_gptq_validation(L):
    """GPTQ's arguments are checked before anything runs (no device needed)."""
    import block_scale_search_b200 as nv
    f = L.nvfp4_gptq_quantize
    ok = dict(W=P, out=64, inp=256, ldw=256, X=P, tokens=128, ldx=256, q=448.0, lo=-9, hi=6,
              damp=0.01, w=1, codes=P, scales=P, S=P, h=P, st=None, ws=P, nb=1 << 30)

    def call(**k):
        a = {**ok, **k}
        return f(a["W"], a["out"], a["inp"], a["ldw"], a["X"], a["tokens"], a["ldx"], a["q"], a["lo"],
                 a["hi"], a["damp"], a["w"], a["codes"], a["scales"], a["S"], a["h"], a["st"], a["ws"],
                 a["nb"], None)

    assert call(W=None) == -1 and call(h=None) == -1 and call(X=None) == -1
    assert call(out=0) == -1 and call(w=2) == -1 and call(damp=-1.0) == -1
    assert call(q=float("inf")) == -1
    assert call(inp=250, ldw=256, ldx=256) == -2            # in % 16
    assert call(ldx=128) == -2                                # ldx < in
    assert call(tokens=1 << 31) == -2                        # beyond the GEMM's int sizes
    assert call(inp=16 * 65536, ldw=16 * 65536, ldx=16 * 65536) == -2   # in / 16 > 65535
    assert call(lo=-10) == -4
    assert call(X=P + 8) == -3 and call(codes=P + 4) == -3 and call(h=P + 4) == -3
    assert call(W=P + 2) == -3 and call(W=P + 8) == -3        # W's rows are read 16 bytes at a time
    assert call(ldw=260) == -3                                # ldw % 8 != 0
    assert call(ws=None) == -7 and call(ws=P + 64) == -3
    assert L.nvfp4_gptq_workspace_size(64, 250, 128) == 0
    ms = (C.c_float * 6)()
    assert L.nvfp4_gptq_set_timing(2) == -1
    assert L.nvfp4_gptq_phase_times(None, 6) == -1 and L.nvfp4_gptq_phase_times(ms, 7) == -1
    assert L.nvfp4_gptq_phase_times(ms, -1) == -1
    assert L.nvfp4_gptq_workspace_size(64, 16 * 65536, 128) == 0
    g = L.nvfp4_scale_sweep_quantize_f32
    assert g(P, 4, 250, 256, None, P, -9, 6, P, P, None) == -2
    assert g(P, 4, 256, 256, None, P, -10, 6, P, P, None) == -4
    assert g(P + 2, 4, 256, 256, None, P, -9, 6, P, P, None) == -3
    assert g(None, 0, 256, 256, None, None, -9, 6, None, None, None) == 0     # empty
    import torch
    if not torch.cuda.is_available():
        assert call() == -6 and L.nvfp4_gptq_workspace_size(64, 256, 128) == 0
