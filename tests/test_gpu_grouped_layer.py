"""nvfp4_quantize_grouped_layer writes exactly what the grouped and batched
calls write: both inputs' per-expert h, every matrix's S, amax and status,
and both batches' codes, scales and offsets -- with one input's diagonal
Hessian streamed beside the other batch's sweep, in whichever order the call
picks (each case runs with the batches passed both ways round).  Needs a
B200."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def nv():
    import block_scale_search_b200 as nv
    nv.lib()
    return nv


def _run_both(nv, W1, W2, X1, X2, offs, lo=-9, hi=6, q_max=448.0, weighted=True):
    """Compare the grouped layer call, with the batches passed in the given
    order, against the grouped and batched calls; returns which batch the
    call swept first (0: W1's, 1: W2's)."""
    E = len(offs) - 1
    off_d = torch.as_tensor(offs, dtype=torch.int64, device=DEV)
    # reference: the grouped and batched calls
    h1 = nv.diag_hessian_grouped(X1, off_d)
    h2 = nv.diag_hessian_grouped(X2, off_d)
    S, amax, status = nv.global_scale_batched(W1 + W2, q_max)
    hs1 = [h1[i % E] for i in range(len(W1))] if weighted else None
    hs2 = [h2[i % E] for i in range(len(W2))] if weighted else None
    n1 = len(W1)
    ref1 = nv.scale_sweep_quantize_batched(W1, hs1, [S[i:i + 1] for i in range(n1)], lo, hi, True)
    ref2 = nv.scale_sweep_quantize_batched(W2, hs2, [S[n1 + i:n1 + i + 1] for i in range(len(W2))],
                                           lo, hi, True)
    torch.cuda.synchronize()
    # one call
    g1 = torch.empty_like(h1)
    g2 = torch.empty_like(h2)
    gS = torch.empty_like(S)
    gA = torch.empty_like(amax)
    gst = torch.empty_like(status)
    outs, d1, d2 = [], [], []
    for b, (Ws, hb) in enumerate(((W1, g1), (W2, g2))):
        for i, W in enumerate(Ws):
            o, n = W.shape
            c = torch.empty(o, n // 2, dtype=torch.uint8, device=DEV)
            sc = torch.empty(o, n // 16, dtype=torch.uint8, device=DEV)
            of = torch.empty(o, n // 16, dtype=torch.int8, device=DEV)
            idx = i if b == 0 else n1 + i
            h = hb[i % E].data_ptr() if weighted else None
            (d1 if b == 0 else d2).append(nv.SweepDesc(W.data_ptr(), o, n, W.stride(0), h,
                                                       gS[idx:idx + 1].data_ptr(), c.data_ptr(),
                                                       sc.data_ptr(), of.data_ptr()))
            outs.append((c, sc, of))
    x1 = nv.GroupedInput(X1.data_ptr(), off_d.data_ptr(), X1.shape[0], X1.shape[1], X1.stride(0),
                         g1.data_ptr())
    x2 = nv.GroupedInput(X2.data_ptr(), off_d.data_ptr(), X2.shape[0], X2.shape[1], X2.stride(0),
                         g2.data_ptr())
    nb = nv.nvfp4_quantize_grouped_layer_workspace_size(d1, d2, x1, x2, E, gS)
    assert nb > 0
    ws = torch.empty(nb, dtype=torch.uint8, device=DEV)
    order = nv.nvfp4_quantize_grouped_layer_order(d1, d2, x1, x2, E, gS, lo, hi)
    nv.nvfp4_quantize_grouped_layer(d1, d2, x1, x2, E, q_max, lo, hi, gS, gA, gst, ws, nb)
    torch.cuda.synchronize()
    assert torch.equal(g1.view(torch.int32), h1.view(torch.int32))
    assert torch.equal(g2.view(torch.int32), h2.view(torch.int32))
    assert torch.equal(gS.view(torch.int32), S.view(torch.int32))
    assert torch.equal(gA.view(torch.int32), amax.view(torch.int32)) and torch.equal(gst, status)
    for got, want in zip(outs, list(ref1) + list(ref2)):
        for a, b in zip(got, want):
            assert torch.equal(a, b)
    return order


def _run_both_orders(nv, W1, W2, X1, X2, offs, **kw):
    """The call with the batches passed either way round; returns the two
    orders it chose."""
    return (_run_both(nv, W1, W2, X1, X2, offs, **kw), _run_both(nv, W2, W1, X2, X1, offs, **kw))


def _moe(E, counts, gu_out, gu_in, seed):
    import workloads
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64).tolist()
    T = offs[-1]
    X1 = workloads.calib(T, gu_in, 1.0, seed, DEV)
    X2 = workloads.calib(T, gu_out, 1.0, seed + 1, DEV)
    W1 = [workloads.weight(gu_out, gu_in, 0.02, 0.001, 10.0, seed + 10 + k, DEV) for k in range(2 * E)]
    W2 = [workloads.weight(gu_in, gu_out, 0.02, 0.001, 10.0, seed + 100 + k, DEV) for k in range(E)]
    return W1, W2, X1, X2, offs


def test_small_moe_layer(nv):
    E = 6
    W1, W2, X1, X2, offs = _moe(E, [700, 0, 3000, 17, 1200, 5000], 768, 2048, 901)
    # the down batch (the smaller input) goes first whichever way it is passed
    assert _run_both_orders(nv, W1, W2, X1, X2, offs) == (1, 0)


def test_small_moe_layer_mse_window(nv):
    E = 4
    W1, W2, X1, X2, offs = _moe(E, [900, 2100, 0, 40], 768, 2048, 931)
    _run_both_orders(nv, W1, W2, X1, X2, offs, lo=-3, hi=7, q_max=256.0, weighted=False)


def test_moe_layer_at_the_benchmarked_size(nv):
    # the 128-expert layer the bench times: gate/up 768x2048, down 2048x768,
    # 262144 tokens routed top-8 with Zipf(1.1) popularity
    import workloads
    wl = workloads.moe_grouped(device=DEV)
    Ws = {m.name: m.make(DEV) for m in wl.matrices}
    X1 = wl.calibs["gu"].make(DEV)
    X2 = wl.calibs["down"].make(DEV)
    E = wl.experts
    W1 = [Ws[f"e{e}.gate"] for e in range(E)] + [Ws[f"e{e}.up"] for e in range(E)]
    W2 = [Ws[f"e{e}.down"] for e in range(E)]
    assert _run_both_orders(nv, W1, W2, X1, X2, wl.calibs["gu"].row_offsets) == (1, 0)


@pytest.mark.parametrize("seed", [5, 6, 7])
def test_random_moe_layers(nv, seed):
    """Random expert counts, routings (with empty experts), widths, windows
    and objectives: the grouped layer call equals the grouped and batched
    calls."""
    rng = np.random.default_rng(seed)
    E = int(rng.integers(1, 10))
    counts = [int(c) if rng.random() > 0.2 else 0 for c in rng.integers(1, 4000, size=E)]
    gu_in = int(rng.choice([512, 1024, 2048]))
    gu_out = int(rng.choice([256, 768, 1040]))
    W1, W2, X1, X2, offs = _moe(E, counts, gu_out, gu_in, 1000 + 37 * seed)
    lo = int(rng.integers(-10, 1))
    hi = int(rng.integers(0, 16 + lo))
    _run_both_orders(nv, W1, W2, X1, X2, offs, lo=lo, hi=hi,
                     q_max=float(rng.choice([256.0, 448.0])), weighted=bool(rng.random() > 0.3))
