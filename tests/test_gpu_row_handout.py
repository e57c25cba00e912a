"""The run-time row hand-out (weight sweep and activation quantizer) writes
the same bytes as the fixed row stride.  A launch recorded into a CUDA graph
keeps the fixed stride, so a graph replay gives the reference bytes; direct
launches of the same shapes lease a counter slot and take rows from it
(checked by reading the slots).  Also: more launches in flight at once, on
as many streams, than there are slots, where a launch waits for its slot's
previous user.  Needs a B200."""
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def nv():
    import block_scale_search_b200 as nv
    nv.lib()
    return nv


def _inputs(out, inp, weighted, seed):
    import workloads
    W = workloads.weight(out, inp, 0.015, 0.001, 10.0, seed, DEV)
    h = None
    if weighted:
        import block_scale_search_b200 as nv
        h = nv.diag_hessian(workloads.calib(1024, inp, 1.5, seed + 1, DEV))
    return W, h


def _alloc(out, inp):
    return (torch.empty(out, inp // 2, dtype=torch.uint8, device=DEV),
            torch.empty(out, inp // 16, dtype=torch.uint8, device=DEV),
            torch.empty(out, inp // 16, dtype=torch.int8, device=DEV))


def _graph_sweep(nv, W, h, S, lo, hi):
    """The sweep launched from a captured graph: the fixed row stride."""
    out, inp = W.shape
    bufs = _alloc(out, inp)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        nv.nvfp4_scale_sweep_quantize(W, out, inp, inp, h, S, lo, hi, *bufs, stream=s)
    g.replay()
    torch.cuda.synchronize()
    del g
    return bufs


SLOTS, WORDS, STRIPS = 64, 258, 256


def _slots(nv):
    """The counter slots, copied to the host: [64, 258] uint32 as int64."""
    from cuda.bindings import runtime as rt
    addr, nbytes = nv.nvfp4_debug_row_counters()
    assert nbytes == SLOTS * WORDS * 4
    t = torch.empty(SLOTS * WORDS, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    err, = rt.cudaMemcpy(t.data_ptr(), addr, nbytes, rt.cudaMemcpyKind.cudaMemcpyDeviceToDevice)
    assert err == rt.cudaError_t.cudaSuccess, err
    return t.cpu().long().reshape(SLOTS, WORDS) & 0xFFFFFFFF


def _served(nv):
    return int(_slots(nv)[:, STRIPS + 1].sum())


SHAPES = [  # (out, in, weighted, lo, hi): K = 16, 11 and a run-time K; odd rows
    (3001, 8192, True, -9, 6),
    (4096, 4096, False, -3, 7),
    (2047, 4096, True, -8, 7),
    (6000, 2048, True, -2, 3),
]


@pytest.mark.parametrize("out,inp,weighted,lo,hi", SHAPES)
def test_handout_matches_fixed_stride(nv, out, inp, weighted, lo, hi):
    W, h = _inputs(out, inp, weighted, 900 + out % 97)
    S, _, _ = nv.global_scale(W)
    n0 = _served(nv)
    ref = _graph_sweep(nv, W, h, S, lo, hi)
    n1 = _served(nv)
    got = _alloc(out, inp)
    nv.nvfp4_scale_sweep_quantize(W, out, inp, inp, h, S, lo, hi, *got)
    torch.cuda.synchronize()
    assert n1 == n0 and _served(nv) == n1 + 1   # graph: fixed stride; direct: a slot
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    sl = _slots(nv)
    assert torch.all(sl[:, :STRIPS + 1] == 0)    # every slot handed back zeroed


def test_small_or_ragged_rows_keep_the_fixed_stride(nv):
    n0 = _served(nv)
    for out, inp in ((256, 1024), (300, 768), (64, 8192)):
        W, h = _inputs(out, inp, True, 31 + out)
        S, _, _ = nv.global_scale(W)
        got = _alloc(out, inp)
        nv.nvfp4_scale_sweep_quantize(W, out, inp, inp, h, S, -9, 6, *got)
    assert _served(nv) == n0


def test_more_launches_in_flight_than_slots(nv):
    mats = []
    for k, (out, inp, weighted, lo, hi) in enumerate([(4096, 4096, True, -9, 6),
                                                      (2048, 8192, False, -3, 7),
                                                      (3000, 2048, True, -8, 7)]):
        W, h = _inputs(out, inp, weighted, 700 + k)
        S, _, _ = nv.global_scale(W)
        mats.append((W, h, S, lo, hi, _graph_sweep(nv, W, h, S, lo, hi)))
    torch.cuda.synchronize()
    n0 = _served(nv)
    n = SLOTS + 16
    streams = [torch.cuda.Stream() for _ in range(n)]
    outs = [_alloc(*mats[i % len(mats)][0].shape) for i in range(n)]
    torch.cuda.synchronize()
    gate = torch.cuda.Event()
    torch.cuda._sleep(1_000_000_000)  # about 0.5 s: every launch below is queued behind it
    gate.record()
    runs = []
    for i in range(n):
        W, h, S, lo, hi, ref = mats[i % len(mats)]
        out, inp = W.shape
        s = streams[i]
        s.wait_event(gate)
        nv.nvfp4_scale_sweep_quantize(W, out, inp, inp, h, S, lo, hi, *outs[i], stream=s)
        runs.append((outs[i], ref))
    torch.cuda.synchronize()
    for bufs, ref in runs:
        for a, b in zip(bufs, ref):
            assert torch.equal(a, b)
    # every launch took a slot: the last 16 waited, on their own streams, for
    # the launches that had their slots before them
    assert _served(nv) - n0 == n
    assert torch.all(_slots(nv)[:, :STRIPS + 1] == 0)


@pytest.mark.parametrize("tokens,inp,lo,hi", [(20011, 2048, -3, 7), (70000, 256, -9, 6)])
def test_activation_rows_from_the_counter(nv, tokens, inp, lo, hi):
    """The activation quantizer takes rows from a leased counter once every
    team would have four rows or more; a graph replay keeps the stride."""
    import workloads
    A = workloads.calib(tokens, inp, 1.5, 41 + tokens % 7, DEV)

    def bufs():
        return (torch.empty(tokens, dtype=torch.float32, device=DEV),
                torch.empty(tokens, inp // 2, dtype=torch.uint8, device=DEV),
                torch.empty(tokens, inp // 16, dtype=torch.uint8, device=DEV),
                torch.empty(tokens, inp // 16, dtype=torch.int8, device=DEV),
                torch.empty(1, dtype=torch.int32, device=DEV))

    ref = bufs()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    n0 = _served(nv)
    with torch.cuda.graph(g, stream=s):
        nv.nvfp4_quantize_activations(A, tokens, inp, inp, 256.0, lo, hi, *ref, stream=s)
    g.replay()
    torch.cuda.synchronize()
    del g
    n1 = _served(nv)
    got = bufs()
    nv.nvfp4_quantize_activations(A, tokens, inp, inp, 256.0, lo, hi, *got)
    torch.cuda.synchronize()
    assert n1 == n0 and _served(nv) == n1 + 1
    assert int(got[4].item()) == 0 and int(ref[4].item()) == 0
    for a, b in zip(got[:4], ref[:4]):
        assert torch.equal(a, b)
    assert torch.all(_slots(nv)[:, :STRIPS + 1] == 0)
