"""Layer-output check (the synthetic analogue of the H-Scale summary's sec. 3
"Validation and integration" comparison of activation loss against Min-Max).

On a synthetic layer whose calibration channels are independent with
lognormal scales, the diagonal of X^T X is the whole second-order term up to
sampling noise, so selecting scales by the h-weighted error should lower the
layer-output error ||X (W - W_hat)^T||^2 against
  * Min-Max / max-abs RTN (window [0, 0]), and
  * plain-MSE ScaleSweep ([-3, +7], h = 1),
while MSE ScaleSweep should lower the plain weight error against Min-Max.
W_hat is decoded by this library's dequantize; the matmul that measures the
output error is only the yardstick.

Also here: the chosen scale is never worse than the max-abs base scale under
the exact evaluator (offset 0 lies in every window)."""
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


def _quantized(nv, W, h, S, lo, hi):
    codes, scales, _ = nv.scale_sweep_quantize(W, h, S, lo, hi)
    return nv.dequantize(codes, scales, S)


@pytest.mark.parametrize("sigma", [1.0, 1.5])
def test_hessian_weighted_scales_lower_the_output_error(nv, sigma):
    import workloads
    W = workloads.weight(1024, 2048, 0.02, 0.001, 10.0, 811, DEV)
    X = workloads.calib(8192, 2048, sigma, 812, DEV)
    h = nv.diag_hessian(X)
    S, _, _ = nv.global_scale(W, 448.0)
    Wf, Xf = W.float(), X.float()
    res = {}
    for name, hh, lo, hi in (("minmax", None, 0, 0), ("mse", None, -3, 7), ("hscale", h, -9, 6)):
        Wq = _quantized(nv, W, hh, S, lo, hi)
        D = Wf - Wq
        res[name] = {"out": float((Xf @ D.T).pow(2).sum()), "w": float(D.pow(2).sum()),
                     "hw": float((D.pow(2) * h).sum())}
    red_h = 1 - res["hscale"]["out"] / res["minmax"]["out"]
    red_m = 1 - res["mse"]["out"] / res["minmax"]["out"]
    print(f"\nsigma={sigma}: activation-loss reduction vs Min-Max: H-Scale {red_h:.1%}, "
          f"MSE {red_m:.1%}; weight-MSE reduction: MSE "
          f"{1 - res['mse']['w'] / res['minmax']['w']:.1%}, H-Scale "
          f"{1 - res['hscale']['w'] / res['minmax']['w']:.1%}")
    assert res["hscale"]["out"] < res["mse"]["out"] < res["minmax"]["out"]
    assert res["mse"]["w"] < res["minmax"]["w"]
    # the weighted objective it minimises is lower than both others'
    assert res["hscale"]["hw"] < min(res["mse"]["hw"], res["minmax"]["hw"])


@pytest.mark.parametrize("lo,hi,weighted", [(-9, 6, True), (-3, 7, False), (-8, 7, True)])
def test_never_worse_than_the_base_scale(orc, nv, lo, hi, weighted):
    """Offset 0 is in every window, so the chosen scale's exact loss never
    exceeds the max-abs base scale's (ScaleSweep summary, retaining the
    status quo).  Checked on every group of a 70B-MLP-shaped slice: the base
    code comes from the GPU's own [0, 0] sweep, the losses from the oracle's
    exact evaluator -- the window's on the GPU's packed bytes, the base's by
    the definition."""
    import workloads
    W = workloads.weight(2048, 8192, 0.015, 0.001, 10.0, 81, DEV)
    X = workloads.calib(8192, 8192, 1.5, 82, DEV)
    h = nv.diag_hessian(X) if weighted else None
    S, _, _ = nv.global_scale(W)
    codes, scales, _ = nv.scale_sweep_quantize(W, h, S, lo, hi)
    _, base, _ = nv.scale_sweep_quantize(W, h, S, 0, 0)
    torch.cuda.synchronize()
    bits = W.cpu().view(torch.uint16).numpy().reshape(-1, 16)
    n = bits.shape[0]
    hh = None
    if weighted:
        hh = np.broadcast_to(h.cpu().numpy().reshape(1, -1, 16), (2048, 512, 16)).reshape(n, 16)
    Sf = float(S.item())
    won = orc.packed_losses(bits, hh, Sf, codes.cpu().numpy().reshape(n, 8),
                            scales.cpu().numpy().reshape(n))
    at_base = orc.group_losses(bits, hh, Sf, base.cpu().numpy().reshape(n))
    assert np.all(won <= at_base), int(np.sum(won > at_base))
    assert np.mean(won < at_base) > 0.3      # and the search does move most groups
