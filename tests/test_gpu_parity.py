"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded input bytes.  Needs a B200 (sm_100a)."""
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
    assert torch.cuda.is_available()
    return nv


def gpu_layer(nv, W, X, q_max, lo, hi, weighted, offsets=True):
    h = nv.diag_hessian(X) if weighted else None
    S, amax, st = nv.global_scale(W, q_max)
    codes, scales, offs = nv.scale_sweep_quantize(W, h, S, lo, hi, want_offsets=offsets)
    torch.cuda.synchronize()
    return h, S, amax, st, codes, scales, offs


def full_matrix_parity(orc, nv, W, X, q_max, lo, hi, weighted, what):
    h, S, amax, st, codes, scales, offs = gpu_layer(nv, W, X, q_max, lo, hi, weighted)
    bits = to_bits(W)
    S_ref, amax_ref, st_ref = orc.global_scale(bits, q_max)
    assert int(st.item()) == 0 and st_ref == 0
    assert np.float32(S.item()) == S_ref and np.float32(amax.item()) == amax_ref, what
    h_np = None
    if weighted:
        h_np = h.cpu().numpy()
        check_h(h_np, orc.parallel_diag_hessian(X.cpu()))
    rc, rs, ro = orc.parallel_sweep_quantize(bits, h_np, float(S_ref), lo, hi)
    gc, gs, go = codes.cpu().numpy(), scales.cpu().numpy(), offs.cpu().numpy()
    w, hh, _, _ = matrix_groups(bits, gc, gs, h_np)
    res = compare_groups(orc, w, hh, float(S_ref), gc.reshape(-1, 8), gs.reshape(-1),
                         rc.reshape(-1, 8), rs.reshape(-1))
    assert_parity(res, what)
    same = (gs == rs)
    assert np.all(go[same] == ro[same]), "offset differs where the code agrees"
    # dequantize: bit-exact with the oracle's decode of the GPU's own bytes
    deq = nv.dequantize(codes, scales, S).cpu().numpy()
    np.testing.assert_array_equal(deq.view(np.uint32), orc.dequantize(gc, gs, float(S_ref)).view(np.uint32))
    return res


def test_single_layer_256x1024(orc, nv):
    import workloads
    wl = workloads.single_layer()
    m = wl.matrices[0]
    W = m.make(DEV)
    X = wl.calibs[m.x_key].make(DEV)
    for run in wl.runs:
        full_matrix_parity(orc, nv, W, X, wl.q_max, run.lo, run.hi, run.weighted, wl.name)


def test_square_layer_4096_both_windows(orc, nv):
    import workloads
    wl = workloads.square_layer()
    m = wl.matrices[0]
    W = m.make(DEV)
    X = wl.calibs[m.x_key].make(DEV)
    for run in wl.runs:
        full_matrix_parity(orc, nv, W, X, wl.q_max, run.lo, run.hi, run.weighted,
                           f"{wl.name} [{run.lo},{run.hi}]")


@pytest.mark.parametrize("lo,hi", [(0, 0), (-15, 0), (0, 15), (-3, 7), (-8, 7), (-9, 6)])
def test_every_window_shape(orc, nv, lo, hi):
    import workloads
    W = workloads.weight(192, 512, 0.02, 0.01, 10.0, 77, DEV)
    X = workloads.calib(333, 512, 1.0, 78, DEV)
    full_matrix_parity(orc, nv, W, X, 448.0, lo, hi, True, f"window [{lo},{hi}]")
    full_matrix_parity(orc, nv, W, X, 256.0, lo, hi, False, f"mse window [{lo},{hi}]")


@pytest.mark.parametrize("out,inp,pad", [(1, 16, 0), (3, 48, 8), (7, 80, 0), (33, 272, 16), (2, 1040, 24)])
def test_ragged_shapes_and_strides(orc, nv, out, inp, pad):
    """Tiny and odd shapes, leading dimensions larger than `in` (including ones
    that force the two-16-byte-load path), and calibration T not a multiple of
    the unroll."""
    import workloads
    base = workloads.weight(out, inp + pad, 0.02, 0.05, 10.0, 1000 + inp, DEV)
    W = base[:, :inp]
    assert W.stride(0) == inp + pad
    Xb = workloads.calib(37, inp + pad, 1.0, 2000 + inp, DEV)
    X = Xb[:, :inp]
    h = nv.diag_hessian(X)
    check_h(h.cpu().numpy(), orc.diag_hessian(X.contiguous().cpu()))
    S, _, _ = nv.global_scale(W, 448.0)
    codes, scales, offs = nv.scale_sweep_quantize(W, h, S, -9, 6, want_offsets=True)
    bits = to_bits(W.contiguous())
    S_ref = orc.global_scale(bits, 448.0)[0]
    assert np.float32(S.item()) == S_ref
    rc, rs, ro = orc.sweep_quantize(bits, h.cpu().numpy(), float(S_ref), -9, 6)
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    w, hh, _, _ = matrix_groups(bits, gc, gs, h.cpu().numpy())
    res = compare_groups(orc, w, hh, float(S_ref), gc, gs, rc, rs)
    assert res["mismatch"] == 0, res


def test_zero_groups_rows_and_matrix(orc, nv):
    W = torch.zeros(64, 256, dtype=torch.bfloat16, device=DEV)
    S, amax, st = nv.global_scale(W)
    assert S.item() == 0.0 and amax.item() == 0.0 and st.item() == 0
    codes, scales, offs = nv.scale_sweep_quantize(W, None, S, -9, 6, want_offsets=True)
    assert not codes.any() and not scales.any() and not offs.any()
    import workloads
    W = workloads.weight(64, 256, 0.02, 0.0, 1.0, 5, DEV)
    W[3] = 0
    W[:, 32:48] = 0
    W[7, 0:16] = -0.0
    S, _, _ = nv.global_scale(W)
    codes, scales, _ = nv.scale_sweep_quantize(W, None, S, -9, 6)
    bits = to_bits(W)
    rc, rs, _ = orc.sweep_quantize(bits, None, float(S.item()), -9, 6)
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    assert not scales[3].any() and not scales[:, 2].any() and scales[7, 0].item() == 0


@pytest.mark.parametrize("weighted", [False, True])
def test_exact_ties_resolve_like_the_definition(orc, nv, weighted):
    """Few-bit weights (small integers times a power of two) and a power-of-two
    S make exact loss ties between different scales common -- octave pairs that
    reconstruct every element alike, and mirror-image errors.  The definition
    breaks them toward the lowest offset; so must the kernel, bit for bit."""
    g = torch.Generator(device=DEV).manual_seed(21)
    ints = torch.randint(-15, 16, (512, 256), generator=g, device=DEV).float()
    scale = 2.0 ** torch.randint(-3, 3, (512, 16, 1), generator=g, device=DEV).float()
    W = (ints.view(512, 16, 16) * scale).view(512, 256).mul(2.0 ** -6).to(torch.bfloat16)
    S = torch.tensor([2.0 ** -10], device=DEV)
    h = None
    if weighted:
        h = (2.0 ** torch.randint(-4, 5, (256,), generator=g, device=DEV).float())
    for lo, hi in ((-9, 6), (-8, 7), (-3, 7)):
        codes, scales, offs = nv.scale_sweep_quantize(W, h, S, lo, hi, want_offsets=True)
        bits = to_bits(W)
        hn = None if h is None else h.cpu().numpy()
        rc, rs, ro = orc.sweep_quantize(bits, hn, 2.0 ** -10, lo, hi)
        gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
        w, hh, _, _ = matrix_groups(bits, gc, gs, hn)
        res = compare_groups(orc, w, hh, 2.0 ** -10, gc, gs, rc, rs)
        assert res["mismatch"] == 0, res
        np.testing.assert_array_equal(offs.cpu().numpy(), ro)


def test_nonfinite_weight_reports_status(nv):
    import workloads
    for bad in (float("nan"), float("inf"), float("-inf")):
        W = workloads.weight(16, 64, 0.02, 0.0, 1.0, 6, DEV)
        W[5, 17] = bad
        S, amax, st = nv.global_scale(W)
        assert st.item() == -5 and np.isnan(S.item())


def test_tiny_and_huge_scales(orc, nv):
    """Denormal-range S (weights near the bf16 minimum normal), and h spanning
    many decades with zero channels: exact power-of-two rescaling keeps the
    decisions those of the definition."""
    import workloads
    W = (workloads.weight(32, 128, 1.0, 0.0, 1.0, 8, DEV).float() * 2.0 ** -120).to(torch.bfloat16)
    S, _, _ = nv.global_scale(W)
    assert 0 < S.item() < 2.0 ** -126
    h = torch.exp(torch.linspace(-60, 60, 128, device=DEV)).float()
    h[::7] = 0
    for hh in (None, h):
        codes, scales, _ = nv.scale_sweep_quantize(W, hh, S, -9, 6)
        bits = to_bits(W)
        hn = None if hh is None else hh.cpu().numpy()
        rc, rs, _ = orc.sweep_quantize(bits, hn, float(S.item()), -9, 6)
        w, hg, _, _ = matrix_groups(bits, codes.cpu().numpy(), scales.cpu().numpy(), hn)
        res = compare_groups(orc, w, hg, float(S.item()), codes.cpu().numpy(), scales.cpu().numpy(), rc, rs)
        assert_parity(res, "tiny S")


def test_diag_hessian_edges(orc, nv):
    import workloads
    X = workloads.calib(1, 64, 1.0, 9, DEV)
    check_h(nv.diag_hessian(X).cpu().numpy(), orc.diag_hessian(X.cpu()))
    X0 = X[:0]
    h0 = torch.arange(64, dtype=torch.float32, device=DEV)
    h = nv.diag_hessian(X0, h0.clone(), accumulate=True)
    assert torch.equal(h, h0)
    assert not nv.diag_hessian(X0).any()
    X = workloads.calib(1000, 64, 1.0, 10, DEV)
    h = nv.diag_hessian(X, h0.clone(), accumulate=True)
    check_h(h.cpu().numpy(), orc.diag_hessian(X.cpu(), h0.cpu().numpy(), accumulate=True))
    ones = torch.ones(4097, 24, dtype=torch.bfloat16, device=DEV)
    assert torch.all(nv.diag_hessian(ones) == 4097)


def test_base_code_rounding_many_values(orc, nv):
    """Window [0,0] returns the base code, so this exercises the device's
    E4M3 round-to-nearest-even of fl32(fl32(a/6)/S) over many magnitudes,
    including values whose quotient lands on E4M3 midpoints."""
    rng = np.random.default_rng(11)
    n = 1 << 16
    a = np.float32(np.exp(rng.uniform(np.log(1e-6), np.log(3.0), n)))
    tab = orc.e4m3_table()
    mids = ((tab[1:-1] + tab[2:]) / 2).astype(np.float32)
    S = np.float32(2.0 ** -7)
    # a = 6 * S * midpoint is exact in bf16 for these few-bit midpoints
    a[: len(mids)] = np.float32(6.0) * S * mids
    g = np.zeros((n, 16), np.float32)
    g[:, 0] = a
    g[:, 1] = -a / 3
    W = torch.from_numpy(g).to(torch.bfloat16).reshape(n // 4, 64).to(DEV)
    Sd = torch.tensor([S], device=DEV)
    _, scales, _ = nv.scale_sweep_quantize(W, None, Sd, 0, 0)
    bits = to_bits(W).reshape(-1, 16)
    ref = np.array([orc.base_code(bits[i], float(S)) for i in range(n)])
    np.testing.assert_array_equal(scales.cpu().numpy().reshape(-1), ref)


def _sampled_matrix_parity(orc, nv, W, h, S, lo, hi, rows, what):
    codes, scales, _ = nv.scale_sweep_quantize(W, h, S, lo, hi)
    ridx = torch.tensor(rows, device=W.device)
    bits = to_bits(W.index_select(0, ridx))
    hn = None if h is None else h.cpu().numpy()
    Sf = float(S.item())
    rc, rs, _ = orc.parallel_sweep_quantize(bits, hn, Sf, lo, hi)
    gc = codes.index_select(0, ridx).cpu().numpy()
    gs = scales.index_select(0, ridx).cpu().numpy()
    w, hh, _, _ = matrix_groups(bits, gc, gs, hn)
    res = compare_groups(orc, w, hh, Sf, gc, gs, rc, rs)
    assert_parity(res, what)
    return res


def _sampled_h_parity(orc, nv, X, h, ncols=48, seed=0):
    rng = np.random.default_rng(seed)
    cols = np.sort(rng.choice(X.shape[1], size=min(ncols, X.shape[1]), replace=False))
    sub = X[:, torch.tensor(cols, device=X.device)].contiguous().cpu()
    check_h(h.cpu().numpy()[cols], orc.diag_hessian(sub))


@pytest.mark.slow
def test_llama3_8b_projections_sampled(orc, nv):
    import workloads
    wl = workloads.llama3_8b()
    hs = {}
    for key, cal in wl.calibs.items():
        X = cal.make(DEV)
        hs[key] = nv.diag_hessian(X)
        _sampled_h_parity(orc, nv, X, hs[key], seed=len(hs))
        del X
    rng = np.random.default_rng(3)
    for m in wl.matrices:
        W = m.make(DEV)
        S, _, _ = nv.global_scale(W, wl.q_max)
        assert np.float32(S.item()) == orc.global_scale(to_bits(W), wl.q_max)[0]
        rows = sorted(rng.choice(m.out, size=min(96, m.out), replace=False).tolist() + [0, m.out - 1])
        _sampled_matrix_parity(orc, nv, W, hs[m.x_key], S, -9, 6, rows, f"{wl.name}.{m.name}")
        del W
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_llama33_70b_mlp_sampled(orc, nv):
    import workloads
    wl = workloads.llama33_70b_mlp()
    hs = {}
    for key, cal in wl.calibs.items():
        X = cal.make(DEV)
        hs[key] = nv.diag_hessian(X)
        _sampled_h_parity(orc, nv, X, hs[key], seed=7 + len(hs))
        del X
        torch.cuda.empty_cache()
    rng = np.random.default_rng(4)
    for m in wl.matrices:
        W = m.make(DEV)
        S, _, _ = nv.global_scale(W, wl.q_max)
        S_ref = orc.global_scale(to_bits(W), wl.q_max)[0]
        assert np.float32(S.item()) == S_ref
        rows = sorted(set(rng.choice(m.out, size=48, replace=False).tolist() + [0, m.out - 1]))
        _sampled_matrix_parity(orc, nv, W, hs[m.x_key], S, -9, 6, rows, f"{wl.name}.{m.name}")
        del W
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_moe_grouped_sampled_experts(orc, nv):
    import workloads
    wl = workloads.moe_grouped(device=DEV)
    offs = wl.calibs["gu"].row_offsets
    counts = np.diff(offs)
    experts = sorted({0, 1, int(np.argmin(counts)), wl.experts - 1, 63})
    Xs = {k: c.make(DEV) for k, c in wl.calibs.items()}
    for e in experts:
        r0, r1 = offs[e], offs[e + 1]
        for m in [mm for mm in wl.matrices if mm.expert == e]:
            X = Xs[m.x_key][r0:r1]
            h = nv.diag_hessian(X)
            check_h(h.cpu().numpy(), orc.parallel_diag_hessian(X.cpu()))
            W = m.make(DEV)
            full_matrix_parity(orc, nv, W, X, wl.q_max, -9, 6, True, m.name)
    del Xs
    torch.cuda.empty_cache()


@pytest.mark.parametrize("weighted", [False, True])
def test_full_sweep_all_126_codes(orc, nv, weighted):
    """The exhaustive sweep over every positive E4M3 code against the oracle's
    sweep over offsets -125..+125 (which clamps to the same 126 codes)."""
    import workloads
    W = workloads.weight(96, 1024, 0.02, 0.01, 10.0, 123, DEV)
    W[5, :48] *= 1e-3  # tiny groups: candidates far below the base code win
    h = nv.diag_hessian(workloads.calib(300, 1024, 1.5, 124, DEV)) if weighted else None
    S, _, _ = nv.global_scale(W)
    codes, scales, offs = nv.scale_sweep_quantize_full(W, h, S, want_offsets=True)
    bits = to_bits(W)
    hn = None if h is None else h.cpu().numpy()
    rc, rs, _ = orc.parallel_sweep_quantize(bits, hn, float(S.item()), -125, 125)
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    w, hh, _, _ = matrix_groups(bits, gc, gs, hn)
    res = compare_groups(orc, w, hh, float(S.item()), gc, gs, rc, rs)
    assert res["mismatch"] == 0, res
    base = np.array([orc.base_code(bits.reshape(-1, 16)[i], float(S.item()))
                     for i in range(bits.size // 16)]).reshape(gs.shape)
    nz = base > 0
    np.testing.assert_array_equal(offs.cpu().numpy()[nz], (gs.astype(int) - base)[nz])
