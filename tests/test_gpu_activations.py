"""GPU parity of the online activation quantizer (ScaleSweep summary, W+A
settings: per-token dynamic global scale, MSE sweep over [-3, +7]) against
the oracle on the same bf16 bytes, through the C ABI.  Needs a B200."""
import numpy as np
import pytest
import torch

from parity import LOSS_RTOL, MATCH_FRACTION, to_bits

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def nv():
    import block_scale_search_b200 as nv
    nv.lib()
    assert torch.cuda.is_available()
    return nv


def act_parity(orc, bits, S_ref, gc, gs, go, rc, rs, ro, what):
    """Per-group match, with mismatched groups scored by the oracle under
    their own row's S; offsets must agree wherever the scale byte does."""
    t, n = bits.shape
    G = n // 16
    gc3, rc3 = gc.reshape(t, G, 8), rc.reshape(t, G, 8)
    match = (gs == rs) & np.all(gc3 == rc3, axis=2)
    worst = 0.0
    for r in np.flatnonzero(~match.all(axis=1)):
        bad = np.flatnonzero(~match[r])
        w = bits[r].reshape(G, 16)[bad]
        lg = orc.packed_losses(w, None, float(S_ref[r]), gc3[r, bad], gs[r, bad])
        lr = orc.packed_losses(w, None, float(S_ref[r]), rc3[r, bad], rs[r, bad])
        rel = np.where(lr > 0, (lg - lr) / np.maximum(lr, 1e-300), np.where(lg > 0, np.inf, 0.0))
        worst = max(worst, float(rel.max()))
    frac = float(match.mean()) if match.size else 1.0
    assert frac >= MATCH_FRACTION, f"{what}: match {frac}"
    assert worst <= LOSS_RTOL, f"{what}: worst relative loss {worst}"
    same = gs == rs
    assert np.all(go[same] == ro[same]), f"{what}: offset differs where the code agrees"
    return frac, worst


def run_pair(orc, nv, A, q_max=256.0, lo=-3, hi=7, what=""):
    S, codes, scales, offs, st = nv.quantize_activations(A, q_max, lo, hi, want_offsets=True)
    torch.cuda.synchronize()
    bits = to_bits(A)
    S_ref, rc, rs, ro, st_ref = orc.parallel_quantize_activations(bits, q_max, lo, hi)
    Sg = S.cpu().numpy()
    np.testing.assert_array_equal(Sg.view(np.uint32), S_ref.view(np.uint32), err_msg=what)
    assert int(st.item()) == st_ref, what
    res = act_parity(orc, bits, S_ref, codes.cpu().numpy(), scales.cpu().numpy(),
                     offs.cpu().numpy(), rc, rs, ro, what)
    return res, (S, codes, scales, offs, st)


@pytest.mark.parametrize("tokens,inp", [(3, 8192), (700, 2048), (6000, 512), (1001, 768),
                                        (17, 14336)])
def test_activation_parity_shapes(orc, nv, tokens, inp):
    """Shapes that select every team size (rows per CTA wave from a few to
    several per warp), ragged token counts and group counts that do not fill
    the last lane stride."""
    import workloads
    A = workloads.calib(tokens, inp, 1.5, 900 + tokens, DEV)
    run_pair(orc, nv, A, what=f"{tokens}x{inp}")


def test_activation_windows_and_q(orc, nv):
    import workloads
    A = workloads.calib(300, 1024, 1.0, 77, DEV, dist="student_t4")
    for q, lo, hi in ((256.0, -3, 7), (448.0, -3, 7), (448.0, -9, 6), (256.0, -8, 7),
                      (256.0, 0, 0), (256.0, -15, 0), (256.0, 0, 15)):
        run_pair(orc, nv, A, q, lo, hi, what=f"q={q} [{lo},{hi}]")


def test_activation_padded_rows(orc, nv):
    """lda > in: the padding is never read (filled with NaN to show it)."""
    import workloads
    base = workloads.calib(257, 1040, 1.0, 31, DEV)
    buf = torch.full((257, 1056), float("nan"), dtype=torch.bfloat16, device=DEV)
    buf[:, :1040] = base
    A = buf[:, :1040]
    assert A.stride(0) == 1056
    (_, _), out = run_pair(orc, nv, A, what="padded")
    assert int(out[4].item()) == 0


def test_activation_edge_rows(orc, nv):
    """Zero rows, rows holding Inf or NaN, tiny rows (S in the FP32 denormal
    range), huge rows, single nonzero elements and negative zeros."""
    import workloads
    A = workloads.calib(12, 512, 1.0, 5, "cpu").to(torch.float32)
    A[1] = 0.0
    A[2, 100] = float("inf")
    A[3, 7] = float("nan")
    A[4] *= 2.0 ** -120
    A[5] *= 2.0 ** 100
    A[6] = 0.0
    A[6, 300] = -3.5
    A[7] = -0.0
    A[8, :256] = 0.0
    A[9] *= 2.0 ** -133
    A = A.to(torch.bfloat16).to(DEV)
    (_, _), (S, codes, scales, offs, st) = run_pair(orc, nv, A, what="edge rows")
    assert int(st.item()) == -5
    Sc = S.cpu().numpy()
    assert Sc[1] == 0 and Sc[7] == 0 and np.isnan(Sc[2]) and np.isnan(Sc[3])
    c, s = codes.cpu().numpy(), scales.cpu().numpy()
    for r in (1, 2, 3, 7):
        assert not c[r].any() and not s[r].any()
    # a clean call afterwards resets the status word
    (_, _), out = run_pair(orc, nv, A[[0, 4, 5]].contiguous(), what="clean rows")
    assert int(out[4].item()) == 0


def test_activation_llama70b_sampled_rows(orc, nv):
    """The 70B-MLP-shaped activation matrix (65536 tokens x 8192, lognormal
    sigma 1.5 channel scales) in the launch configuration the benchmark times;
    rows are independent, so sampled rows are checked against the oracle
    computed on those rows alone."""
    import workloads
    A = workloads.calib(65536, 8192, 1.5, 4, DEV)
    S, codes, scales, offs, st = nv.quantize_activations(A, 256.0, -3, 7, want_offsets=True)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g = torch.Generator().manual_seed(11)
    rows = torch.cat([torch.tensor([0, 1, 2959, 2960, 65535]),
                      torch.randint(0, 65536, (251,), generator=g)]).unique()
    sub = A[rows.to(DEV)].contiguous()
    bits = to_bits(sub)
    S_ref, rc, rs, ro, st_ref = orc.parallel_quantize_activations(bits, 256.0, -3, 7)
    assert st_ref == 0
    Sg = S[rows.to(DEV)].cpu().numpy()
    np.testing.assert_array_equal(Sg.view(np.uint32), S_ref.view(np.uint32))
    ridx = rows.to(DEV)
    act_parity(orc, bits, S_ref, codes[ridx].cpu().numpy(), scales[ridx].cpu().numpy(),
               offs[ridx].cpu().numpy(), rc, rs, ro, "70B activations, sampled rows")


def test_activation_repeatable(nv):
    import workloads
    A = workloads.calib(2000, 4096, 1.0, 8, DEV)
    a = nv.quantize_activations(A, want_offsets=True)
    b = nv.quantize_activations(A, want_offsets=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8) if x.dtype == torch.float32 else x,
                           y.view(torch.uint8) if y.dtype == torch.float32 else y)
