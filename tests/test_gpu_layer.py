"""nvfp4_quantize_layer writes exactly what the per-step calls write: h of
every input, S (and status) of every weight, codes, scales and offsets of
every sweep -- whether the reductions ride along earlier sweeps (shapes whose
rows hold a multiple of 512 elements, long enough to hand rows out at run
time) or run on their own.  Needs a B200."""
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


def _per_step(nv, Ws, Xs, inputs, q_max, lo, hi):
    hs = [nv.diag_hessian(X) for X in Xs]
    res = []
    for W, k in zip(Ws, inputs):
        S, _, st = nv.global_scale(W, q_max)
        h = hs[k] if k >= 0 else None
        codes, scales, offs = nv.scale_sweep_quantize(W, h, S, lo, hi, want_offsets=True)
        res.append((codes, scales, S, offs, st))
    torch.cuda.synchronize()
    return res, hs


def _check_same(nv, Ws, Xs, inputs, q_max=448.0, lo=-9, hi=6):
    ref, href = _per_step(nv, Ws, Xs, inputs, q_max, lo, hi)
    got, hgot = nv.quantize_layer_many(Ws, Xs, inputs, q_max, lo, hi, want_offsets=True)
    torch.cuda.synchronize()
    for a, b in zip(hgot, href):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    for (c, s, S, o, st), (rc, rs, rS, ro, rst) in zip(got, ref):
        assert torch.equal(S.view(torch.int32), rS.view(torch.int32))
        assert int(st.item()) == int(rst.item())
        assert torch.equal(c, rc) and torch.equal(s, rs) and torch.equal(o, ro)


def _mlp(gu_out, gu_in, down_out, tokens, seed):
    import workloads
    Ws = [workloads.weight(gu_out, gu_in, 0.015, 0.001, 10.0, seed, DEV),
          workloads.weight(gu_out, gu_in, 0.015, 0.001, 10.0, seed + 1, DEV),
          workloads.weight(down_out, gu_out, 0.015, 0.001, 10.0, seed + 2, DEV)]
    Xs = [workloads.calib(tokens, gu_in, 1.5, seed + 3, DEV),
          workloads.calib(tokens, gu_out, 1.5, seed + 4, DEV)]
    return Ws, Xs, [0, 0, 1]


def test_mlp_with_reductions_carried(nv):
    # gate/up 3072x2048 and down 2048x3072: both gate and up carry side work
    Ws, Xs, inputs = _mlp(3072, 2048, 2048, 4096, 11)
    _check_same(nv, Ws, Xs, inputs)


def test_mlp_at_the_benchmarked_size(nv):
    # the 70B-shaped MLP the bench times: gate/up 28672x8192, down 8192x28672,
    # 65536 calibration tokens per input
    Ws, Xs, inputs = _mlp(28672, 8192, 8192, 65536, 4)
    _check_same(nv, Ws, Xs, inputs)


def test_small_or_ragged_shapes_run_on_their_own(nv):
    # rows too short or not a multiple of 512 elements: nothing rides along
    Ws, Xs, inputs = _mlp(256, 768, 96, 300, 21)
    _check_same(nv, Ws, Xs, inputs)


def test_mse_weights_shared_and_unused_inputs(nv):
    import workloads
    Ws = [workloads.weight(3000, 4096, 0.02, 0.001, 8.0, 31, DEV),   # MSE, first
          workloads.weight(4096, 4096, 0.02, 0.001, 8.0, 32, DEV),   # input 1
          workloads.weight(2500, 4096, 0.02, 0.001, 8.0, 33, DEV),   # input 1 again
          workloads.weight(4096, 2048, 0.02, 0.001, 8.0, 34, DEV)]   # input 2
    Xs = [workloads.calib(512, 1024, 1.0, 35, DEV),                   # used by no weight
          workloads.calib(2048, 4096, 1.0, 36, DEV),
          workloads.calib(3000, 2048, 1.0, 37, DEV)]
    _check_same(nv, Ws, Xs, [-1, 1, 1, 2], q_max=256.0, lo=-3, hi=7)
    _check_same(nv, Ws, Xs, [-1, 1, 1, 2], q_max=448.0, lo=-8, hi=7)


def test_nonfinite_weight_reports_its_own_status(nv):
    Ws, Xs, inputs = _mlp(3072, 2048, 2048, 2048, 41)
    Ws[1][5, 7] = float("inf")   # up: its S is carried by the gate sweep
    Ws[2][9, 3] = float("nan")   # down
    got, _ = nv.quantize_layer_many(Ws, Xs, inputs)
    torch.cuda.synchronize()
    assert [int(g[4].item()) for g in got] == [0, -5, -5]
    assert torch.isnan(got[1][2]).all() and torch.isnan(got[2][2]).all()


def test_layer_call_captured_in_a_graph(nv):
    """Under stream capture no sweep can take a counter slot: every sweep
    keeps the fixed stride and every reduction runs on its own; a replay
    writes the same bytes as the per-step calls."""
    Ws, Xs, inputs = _mlp(3072, 2048, 2048, 4096, 51)
    ref, href = _per_step(nv, Ws, Xs, inputs, 448.0, -9, 6)
    got = []
    hs = [torch.empty(X.shape[1], dtype=torch.float32, device=DEV) for X in Xs]
    wd = []
    for W, k in zip(Ws, inputs):
        o, n = W.shape
        t = (torch.empty(o, n // 2, dtype=torch.uint8, device=DEV),
             torch.empty(o, n // 16, dtype=torch.uint8, device=DEV),
             torch.empty(1, dtype=torch.float32, device=DEV),
             torch.empty(o, n // 16, dtype=torch.int8, device=DEV),
             torch.empty(1, dtype=torch.int32, device=DEV))
        got.append(t)
        wd.append(nv.LayerWeight(W.data_ptr(), o, n, W.stride(0), k, t[2].data_ptr(), None,
                                 t[4].data_ptr(), t[0].data_ptr(), t[1].data_ptr(), t[3].data_ptr()))
    xd = [nv.LayerInput(X.data_ptr(), X.shape[0], X.shape[1], X.stride(0), h.data_ptr())
          for X, h in zip(Xs, hs)]
    nb = nv.nvfp4_quantize_layer_workspace_size(wd, xd)
    ws = torch.empty(nb, dtype=torch.uint8, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        nv.nvfp4_quantize_layer(wd, xd, 448.0, -9, 6, ws, nb, stream=s)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    del g
    for a, b in zip(hs, href):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    for (c, sc, S, o, st), (rc, rs, rS, ro, rst) in zip(got, ref):
        assert torch.equal(S.view(torch.int32), rS.view(torch.int32)) and int(st.item()) == 0
        assert torch.equal(c, rc) and torch.equal(sc, rs) and torch.equal(o, ro)


def test_many_projections_fill_the_side_job_slots(nv):
    """Twelve weights over four inputs: later sweeps have up to eleven earlier
    carriers and a sweep can carry at most eight reductions at once, so the
    planner both spreads and caps; the bytes are still the per-step calls'."""
    import workloads
    shapes = [(4096, 2048, 0), (3072, 2048, 0), (2048, 4096, 1), (4096, 4096, 1),
              (2560, 2048, 2), (3000, 4096, 1), (2048, 2048, 3), (4096, 2048, 0),
              (2048, 4096, -1), (3072, 2048, 2), (2048, 2048, 3), (2600, 4096, 1)]
    Ws = [workloads.weight(o, i, 0.02, 0.001, 10.0, 600 + k, DEV) for k, (o, i, _) in enumerate(shapes)]
    Xs = [workloads.calib(2048, 2048, 1.0, 650, DEV), workloads.calib(1536, 4096, 1.0, 651, DEV),
          workloads.calib(3000, 2048, 1.0, 652, DEV), workloads.calib(1024, 2048, 1.0, 653, DEV)]
    _check_same(nv, Ws, Xs, [k for _, _, k in shapes])


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_random_layers(nv, seed):
    """Random projections over random inputs (shapes a multiple of 16 wide,
    some long enough to carry side work, some not; weighted and MSE weights;
    random windows): the layer call equals the per-step calls."""
    import workloads
    rng = np.random.default_rng(seed)
    nx = int(rng.integers(1, 4))
    widths = [int(rng.choice([512, 1024, 2048, 4096, 1040])) for _ in range(nx)]
    Xs = [workloads.calib(int(rng.integers(1, 3000)), w, 1.0, 700 + 10 * seed + k, DEV)
          for k, w in enumerate(widths)]
    nw = int(rng.integers(1, 7))
    Ws, inputs = [], []
    for j in range(nw):
        k = int(rng.integers(-1, nx))
        inp = widths[k] if k >= 0 else int(rng.choice([256, 2048]))
        out = int(rng.choice([64, 700, 3000, 5000]))
        Ws.append(workloads.weight(out, inp, 0.02, 0.001, 10.0, 800 + 10 * seed + j, DEV))
        inputs.append(k)
    lo = int(rng.integers(-12, 1))
    hi = int(rng.integers(0, 16 + lo))
    _check_same(nv, Ws, Xs, inputs, q_max=float(rng.choice([256.0, 448.0])), lo=lo, hi=hi)


def _order(nv, Ws, Xs, inputs, lo=-9, hi=6):
    """The sweep order the layer call picks for these shapes (descriptors
    with placeholder outputs; nothing is launched)."""
    wd = [nv.LayerWeight(W.data_ptr(), *W.shape, W.stride(0), k, W.data_ptr(), None, None,
                         W.data_ptr(), W.data_ptr(), None) for W, k in zip(Ws, inputs)]
    xd = [nv.LayerInput(X.data_ptr(), *X.shape, X.stride(0), X.data_ptr()) for X in Xs]
    return nv.nvfp4_quantize_layer_order(wd, xd, lo, hi)


def test_sweep_order_is_chosen_and_writes_the_same_bytes(nv):
    """The call sweeps the weights in the order with the lowest estimated time.
    Given gate, up, down, it keeps that order. Given down first, it sweeps a
    projection reading the smaller gate/up input first, and writes the per-step
    calls' bytes all the same."""
    Ws, Xs, inputs = _mlp(3072, 2048, 2048, 4096, 31)
    assert _order(nv, Ws, Xs, inputs) == [0, 1, 2]
    given = [2, 0, 1]                      # down, gate, up
    Ws2 = [Ws[i] for i in given]
    in2 = [inputs[i] for i in given]
    o2 = _order(nv, Ws2, Xs, in2)
    assert sorted(o2) == [0, 1, 2] and o2[0] in (1, 2)
    _check_same(nv, Ws2, Xs, in2)
    # and at the benchmarked size, in the bench's order
    Wb, Xb, ib = _mlp(28672, 8192, 8192, 65536, 4)
    assert _order(nv, Wb, Xb, ib) == [0, 1, 2]
    assert _order(nv, [Wb[2], Wb[0], Wb[1]], Xb, [1, 0, 0])[0] in (1, 2)


def test_two_layers_in_one_call(orc, nv):
    """nvfp4_quantize_layers: two MLP layers in one call (the second layer's h
    and S streamed beside the first layer's sweeps) write the per-step calls'
    bytes, and every group matches the oracle fed the same h."""
    from parity import assert_parity, check_h, compare_groups, matrix_groups, to_bits
    layers = [_mlp(3072, 2048, 2048, 4096, 51), _mlp(3072, 2048, 2048, 4096, 61)]
    got = nv.quantize_layers_many(layers, want_offsets=True)
    torch.cuda.synchronize()
    for (Ws, Xs, inputs), (outs, hs) in zip(layers, got):
        ref, href = _per_step(nv, Ws, Xs, inputs, 448.0, -9, 6)
        for a, b, X in zip(hs, href, Xs):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32))
            check_h(a.cpu().numpy(), orc.parallel_diag_hessian(X.cpu()))
        for W, k, (c, s, S, o, st), (rc, rs, rS, ro, rst) in zip(Ws, inputs, outs, ref):
            assert torch.equal(S.view(torch.int32), rS.view(torch.int32)) and int(st.item()) == 0
            assert torch.equal(c, rc) and torch.equal(s, rs) and torch.equal(o, ro)
            bits = to_bits(W)
            h = hs[k].cpu().numpy()
            rcodes, rscales, _ = orc.parallel_sweep_quantize(bits, h, float(S.item()), -9, 6)
            gc, gs = c.cpu().numpy(), s.cpu().numpy()
            w, hh, _, _ = matrix_groups(bits, gc, gs, h)
            assert_parity(compare_groups(orc, w, hh, float(S.item()), gc, gs, rcodes, rscales))


def test_layers_with_mse_weights_and_unused_inputs(nv):
    """nvfp4_quantize_layers over layers of different make-up -- a plain-MSE
    weight, an input no weight reads, a layer of one weight -- writes the
    per-step calls' bytes."""
    import workloads
    L1 = ([workloads.weight(2048, 4096, 0.02, 0.001, 8.0, 111, DEV),
           workloads.weight(1536, 4096, 0.02, 0.001, 8.0, 112, DEV)],
          [workloads.calib(1024, 1024, 1.0, 113, DEV), workloads.calib(2048, 4096, 1.0, 114, DEV)],
          [-1, 1])
    L2 = ([workloads.weight(4096, 2048, 0.02, 0.001, 8.0, 121, DEV)],
          [workloads.calib(3000, 2048, 1.0, 122, DEV)], [0])
    got = nv.quantize_layers_many([L1, L2], q_max=256.0, lo=-8, hi=7, want_offsets=True)
    torch.cuda.synchronize()
    for (Ws, Xs, inputs), (outs, hs) in zip([L1, L2], got):
        ref, href = _per_step(nv, Ws, Xs, inputs, 256.0, -8, 7)
        for a, b in zip(hs, href):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32))
        for (c, s, S, o, st), (rc, rs, rS, ro, rst) in zip(outs, ref):
            assert torch.equal(S.view(torch.int32), rS.view(torch.int32))
            assert torch.equal(c, rc) and torch.equal(s, rs) and torch.equal(o, ro)
