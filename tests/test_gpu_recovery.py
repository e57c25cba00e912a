"""Window recovery and scale-direction statistics (synthetic analogues of the
H-Scale summary's sec. 4 ablations: recovery of the full search's gain as the
number of upward steps U grows, and how often the chosen scale is larger,
equal to or smaller than the max-abs initialisation).

Per group, with L the h-weighted loss of the decoded weights:
  recovery(window) = (L_base - L_window) / (L_base - L_full)
over groups the full 126-code sweep improves.  Structural facts are asserted
(the full sweep is never beaten; recovery grows with U); the table is printed."""
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


def _group_losses(nv, W, h, S, codes, scales):
    Wq = nv.dequantize(codes, scales, S).double()
    D = (W.double() - Wq) ** 2 * h.double()
    return D.view(W.shape[0], -1, 16).sum(-1).reshape(-1)


def test_window_recovery_and_direction(nv):
    import workloads
    W = workloads.weight(4096, 8192, 0.015, 0.001, 10.0, 901, DEV)
    X = workloads.calib(8192, 8192, 1.5, 902, DEV)
    h = nv.diag_hessian(X)
    S, _, _ = nv.global_scale(W)
    c, s, _ = nv.scale_sweep_quantize(W, h, S, 0, 0)
    L_base = _group_losses(nv, W, h, S, c, s)
    c, s, _ = nv.scale_sweep_quantize_full(W, h, S)
    L_full = _group_losses(nv, W, h, S, c, s)
    gain = L_base - L_full
    sel = gain > 1e-12 * L_base.clamp_min(1e-300)
    assert torch.all(L_full <= L_base * (1 + 1e-9))
    rows = []
    med_prev = -1.0
    for U in range(0, 8):
        lo = max(-9, U - 15)
        c, s, offs = nv.scale_sweep_quantize(W, h, S, lo, U, want_offsets=True)
        L = _group_losses(nv, W, h, S, c, s)
        assert torch.all(L >= L_full * (1 - 1e-9))
        rec = ((L_base - L) / gain)[sel].cpu().numpy()
        med, p10 = float(np.median(rec)), float(np.percentile(rec, 10))
        exact = float((L[sel] <= L_full[sel] * (1 + 1e-9)).float().mean())
        rows.append((lo, U, med, p10, exact))
        assert med >= med_prev - 1e-9
        med_prev = med
    c, s, offs = nv.scale_sweep_quantize(W, h, S, -9, 6, want_offsets=True)
    o = offs.cpu().numpy().reshape(-1)
    larger, same, smaller = (o > 0).mean(), (o == 0).mean(), (o < 0).mean()
    removed = 1 - float(L_full.sum() / L_base.sum())
    removed96 = 1 - float(_group_losses(nv, W, h, S, c, s).sum() / L_base.sum())
    print("\nwindow  median-recovery  P10-recovery  groups-at-full-optimum")
    for lo, U, med, p10, exact in rows:
        print(f"[{lo:+d},{U:+d}]  {med:14.2%}  {p10:12.2%}  {exact:12.2%}")
    print(f"full 126-code sweep removes {removed:.1%} of the max-abs error; [-9,+6] removes "
          f"{removed96:.1%}")
    print(f"direction vs max-abs ([-9,+6]): larger {larger:.1%}, same {same:.1%}, smaller {smaller:.1%}")
    assert removed96 <= removed + 1e-9 and removed96 > 0
