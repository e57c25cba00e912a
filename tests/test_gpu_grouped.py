"""Grouped diagonal Hessian and batched global scale / sweep on a B200:
identical results to the single-matrix calls (bit for bit for S and the
sweep), and parity with the CPU oracle on ragged expert slices."""
import numpy as np
import pytest
import torch

from parity import assert_parity, check_h, compare_groups, matrix_groups, to_bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def nv():
    import block_scale_search_b200 as nv
    nv.lib()
    return nv


@pytest.mark.parametrize("inp", [768, 2048, 64])
def test_grouped_diag_hessian_ragged_experts(orc, nv, inp):
    """Experts with 0, 1, fewer and more tokens than one chunk, and a long one."""
    import workloads
    counts = [0, 1, 37, 512, 513, 0, 1500, 2, 1024, 7]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    T = int(offs[-1])
    X = workloads.calib(T, inp, 1.0, 61 + inp, DEV)
    off_d = torch.from_numpy(offs).to(DEV)
    h = nv.diag_hessian_grouped(X, off_d)
    Xc = X.cpu()
    for e in range(len(counts)):
        sub = Xc[offs[e]:offs[e + 1]]
        check_h(h[e].cpu().numpy(), orc.diag_hessian(sub))
        if counts[e] == 0:
            assert not h[e].any()
    # accumulate adds onto the previous values
    h2 = nv.diag_hessian_grouped(X, off_d, h.clone(), accumulate=True)
    np.testing.assert_allclose(h2.cpu().numpy(), 2 * h.cpu().numpy(), rtol=2e-7)


def test_grouped_equals_per_expert_single_calls(nv):
    import workloads
    counts = [300, 0, 2100, 64]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    X = workloads.calib(int(offs[-1]), 2048, 1.5, 71, DEV)
    hg = nv.diag_hessian_grouped(X, torch.from_numpy(offs).to(DEV))
    for e, c in enumerate(counts):
        hs = nv.diag_hessian(X[offs[e]:offs[e + 1]])
        np.testing.assert_allclose(hg[e].cpu().numpy(), hs.cpu().numpy(), rtol=1e-5)


def _mixed_matrices():
    import workloads
    shapes = [(768, 2048), (2048, 768), (1, 16), (33, 272), (512, 4096), (0, 64), (2, 1040)]
    Ws = []
    for k, (o, i) in enumerate(shapes):
        if o == 0:
            Ws.append(torch.empty(0, i, dtype=torch.bfloat16, device=DEV))
        else:
            Ws.append(workloads.weight(o, i, 0.02, 0.002, 10.0, 90 + k, DEV))
    return Ws


def test_batched_global_scale_equals_single_calls(nv):
    Ws = _mixed_matrices()
    Ws[3][5, 7] = float("inf")
    S, amax, st = nv.global_scale_batched(Ws, 448.0)
    for i, W in enumerate(Ws):
        if W.numel() == 0:
            assert S[i].item() == 0 and st[i].item() == 0
            continue
        s1, a1, t1 = nv.global_scale(W, 448.0)
        assert t1.item() == st[i].item()
        if t1.item() == 0:
            assert S[i].item() == s1.item() and amax[i].item() == a1.item()
        else:
            assert np.isnan(S[i].item())


@pytest.mark.parametrize("weighted,lo,hi", [(True, -9, 6), (False, -3, 7), (True, -8, 7)])
def test_batched_sweep_bit_identical_to_single_calls(nv, weighted, lo, hi):
    import workloads
    Ws = [W for W in _mixed_matrices()]
    S, _, _ = nv.global_scale_batched(Ws, 448.0)
    hs = None
    if weighted:
        hs = [nv.diag_hessian(workloads.calib(97, W.shape[1], 1.0, 140 + i, DEV)) for i, W in enumerate(Ws)]
    outs = nv.scale_sweep_quantize_batched(Ws, hs, [S[i:i + 1] for i in range(len(Ws))], lo, hi,
                                           want_offsets=True)
    for i, W in enumerate(Ws):
        if W.numel() == 0:
            continue
        c1, s1, o1 = nv.scale_sweep_quantize(W, None if hs is None else hs[i], S[i:i + 1], lo, hi,
                                             want_offsets=True)
        assert torch.equal(outs[i][0], c1) and torch.equal(outs[i][1], s1) and torch.equal(outs[i][2], o1)


@pytest.mark.slow
def test_moe_layer_through_grouped_calls(orc, nv):
    """The whole MoE-shaped layer through the grouped/batched entry points:
    per-expert h from one launch per calibration tensor, 384 global scales in
    one launch, 384 sweeps in one launch; sampled experts against the oracle."""
    import workloads
    wl = workloads.moe_grouped(device=DEV)
    offs = wl.calibs["gu"].row_offsets
    off_d = torch.tensor(offs, dtype=torch.int64, device=DEV)
    h = {}
    for key, cal in wl.calibs.items():
        X = cal.make(DEV)
        h[key] = nv.diag_hessian_grouped(X, off_d)
        del X
    torch.cuda.empty_cache()
    Ws = [m.make(DEV) for m in wl.matrices]
    S, _, st = nv.global_scale_batched(Ws, wl.q_max)
    assert not st.any()
    hs = [h[m.x_key][m.expert] for m in wl.matrices]
    outs = nv.scale_sweep_quantize_batched(Ws, hs, [S[i:i + 1] for i in range(len(Ws))], -9, 6)
    counts = np.diff(offs)
    experts = sorted({0, int(np.argmin(counts)), int(np.argmax(counts)), wl.experts - 1})
    for i, m in enumerate(wl.matrices):
        if m.expert not in experts:
            continue
        bits = to_bits(Ws[i])
        S_ref = orc.global_scale(bits, wl.q_max)[0]
        assert np.float32(S[i].item()) == S_ref
        hn = hs[i].cpu().numpy()
        rc, rs, _ = orc.parallel_sweep_quantize(bits, hn, float(S_ref), -9, 6)
        gc, gs = outs[i][0].cpu().numpy(), outs[i][1].cpu().numpy()
        w, hh, _, _ = matrix_groups(bits, gc, gs, hn)
        assert_parity(compare_groups(orc, w, hh, float(S_ref), gc, gs, rc, rs), m.name)


def test_batched_calls_refuse_stream_capture(nv):
    """The batched S, batched sweep and grouped layer calls stage host tables,
    which a graph replay could not read: on a capturing stream they return
    NVFP4_ERR_CAPTURE and enqueue nothing; the capture itself stays usable."""
    import workloads
    Ws = [workloads.weight(64, 256, 0.02, 0.0, 1.0, 70 + i, DEV) for i in range(2)]
    mdesc = [nv.MatrixDesc(W.data_ptr(), 64, 256, 256) for W in Ws]
    S = torch.zeros(2, device=DEV)
    amax = torch.zeros(2, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    gws = torch.empty(nv.nvfp4_global_scale_batched_workspace_size(mdesc), dtype=torch.uint8,
                      device=DEV)
    codes = [torch.empty(64, 128, dtype=torch.uint8, device=DEV) for _ in Ws]
    scales = [torch.empty(64, 16, dtype=torch.uint8, device=DEV) for _ in Ws]
    sdesc = [nv.SweepDesc(W.data_ptr(), 64, 256, 256, None, S[i:i + 1].data_ptr(),
                          codes[i].data_ptr(), scales[i].data_ptr(), None) for i, W in enumerate(Ws)]
    sws = torch.empty(nv.nvfp4_scale_sweep_quantize_batched_workspace_size(2), dtype=torch.uint8,
                      device=DEV)
    X = workloads.calib(32, 256, 1.0, 72, DEV)
    off = torch.tensor([0, 16, 32], dtype=torch.int64, device=DEV)
    h1 = torch.empty(2, 256, device=DEV)
    h2 = torch.empty(2, 256, device=DEV)
    x1 = nv.GroupedInput(X.data_ptr(), off.data_ptr(), 32, 256, 256, h1.data_ptr())
    x2 = nv.GroupedInput(X.data_ptr(), off.data_ptr(), 32, 256, 256, h2.data_ptr())
    gl = [nv.SweepDesc(W.data_ptr(), 64, 256, 256, h1[i].data_ptr(), S[i:i + 1].data_ptr(),
                       codes[i].data_ptr(), scales[i].data_ptr(), None) for i, W in enumerate(Ws)]
    nb = nv.nvfp4_quantize_grouped_layer_workspace_size(gl[:1], gl[1:], x1, x2, 2, S)
    lws = torch.empty(nb, dtype=torch.uint8, device=DEV)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    got = []
    with torch.cuda.graph(g, stream=s):
        for call in (lambda: nv.nvfp4_global_scale_batched(mdesc, 448.0, S, amax, status, gws,
                                                           gws.numel(), s),
                     lambda: nv.nvfp4_scale_sweep_quantize_batched(sdesc, -9, 6, sws, sws.numel(),
                                                                   s),
                     lambda: nv.nvfp4_quantize_grouped_layer(gl[:1], gl[1:], x1, x2, 2, 448.0, -9,
                                                             6, S, amax, status, lws, nb,
                                                             stream=s)):
            try:
                call()
                got.append(0)
            except nv.NVFP4Error as e:
                got.append(e.status)
        S.add_(1.0)  # the capture goes on after the refusals
    assert got == [-8, -8, -8]
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(S.cpu(), torch.ones(2))
