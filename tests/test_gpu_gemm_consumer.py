"""The packed output is consumable as it is: a Blackwell block-scaled NVFP4
GEMM (cuBLASLt through torch's scaled_mm) reads this library's codes, with
the scales rewritten by nvfp4_scales_to_blocked, and reproduces the product
of the decoded matrices.  Needs a B200."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def nv():
    import block_scale_search_b200 as nv
    nv.lib()
    assert torch.cuda.is_available()
    return nv


def blocked_reference(sf: np.ndarray) -> np.ndarray:
    """The tiled layout written out from its definition, one byte at a time."""
    rows, cols = sf.shape
    rp, cp = -(-rows // 128) * 128, -(-cols // 4) * 4
    out = np.zeros(rp * cp, np.uint8)
    for r in range(rows):
        for c in range(cols):
            blk = (r // 128) * (cp // 4) + c // 4
            rr, cc = r % 128, c % 4
            out[blk * 512 + (rr % 32) * 16 + (rr // 32) * 4 + cc] = sf[r, c]
    return out


@pytest.mark.parametrize("rows,cols", [(1, 1), (128, 4), (300, 130), (257, 7), (513, 512)])
def test_blocked_layout(nv, rows, cols):
    g = torch.Generator().manual_seed(rows * 1000 + cols)
    sf = torch.randint(0, 256, (rows, cols + 3), generator=g, dtype=torch.uint8)
    sfd = sf.to(DEV)[:, :cols]                      # ld = cols + 3
    got = nv.scales_to_blocked(sfd).cpu().numpy()
    exp = blocked_reference(sf[:, :cols].numpy())
    np.testing.assert_array_equal(got, exp)


def _scaled_mm_nvfp4(nv, codes_a, scales_a, sa, codes_b, scales_b, sb, out_dtype):
    import torch.nn.functional as F
    bw, tw = F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise
    sw = F.SwizzleType.SWIZZLE_32_4_4
    ba = nv.scales_to_blocked(scales_a).view(torch.float8_e4m3fn)
    bb = nv.scales_to_blocked(scales_b).view(torch.float8_e4m3fn)
    return F.scaled_mm(codes_a.view(torch.float4_e2m1fn_x2),
                       codes_b.view(torch.float4_e2m1fn_x2).t(),
                       [ba, sa.reshape(1)], [bw, tw], [bb, sb.reshape(1)], [bw, tw],
                       swizzle_a=[sw], swizzle_b=[sw], output_dtype=out_dtype)


def _check(out, ref, absprod):
    # products of decoded values are exact; the GEMM sums them in FP32 and
    # rounds once to bf16 at the end
    err = (out.double() - ref).abs()
    bound = 2.0 ** -8 * ref.abs() + 2.0 ** -16 * absprod + 1e-30
    worst = float((err / bound).max())
    assert worst <= 1.0, f"worst error / bound = {worst:.3g}"
    rel = float(err.norm() / ref.norm())
    assert rel < 4e-3, rel
    return rel


def test_gemm_consumes_weights_and_tensor_scaled_activations(nv):
    """W: the H-Scale sweep ([-9,+6], h from calibration X); A: one S for the
    tensor and the plain-MSE sweep [-3,+7]."""
    import workloads
    M, N, K = 256, 512, 2048
    W = workloads.weight(N, K, 0.02, 0.001, 10.0, 61, DEV)
    X = workloads.calib(4096, K, 1.0, 62, DEV)
    A = workloads.calib(M, K, 1.0, 63, DEV)
    cw, sw_, Sw, _ = nv.quantize_layer(W, X)
    Sa, _, _ = nv.global_scale(A, 448.0)
    ca, sa_, _ = nv.scale_sweep_quantize(A, None, Sa, -3, 7)
    out = _scaled_mm_nvfp4(nv, ca, sa_, Sa, cw, sw_, Sw, torch.bfloat16)
    da = nv.dequantize(ca, sa_, Sa).double()
    dw = nv.dequantize(cw, sw_, Sw).double()
    _check(out, da @ dw.T, da.abs() @ dw.abs().T)


def test_gemm_consumes_per_token_activations(nv):
    """A quantized online, one S per token: the GEMM runs with unit tensor
    scale for A and its output rows are scaled by S_t afterwards."""
    import workloads
    M, N, K = 384, 256, 4096
    W = workloads.weight(N, K, 0.02, 0.001, 10.0, 71, DEV)
    X = workloads.calib(2048, K, 1.5, 72, DEV)
    A = workloads.calib(M, K, 1.5, 73, DEV)
    cw, sw_, Sw, _ = nv.quantize_layer(W, X)
    St, ca, sa_, _, st = nv.quantize_activations(A)
    assert int(st.item()) == 0
    one = torch.ones(1, dtype=torch.float32, device=DEV)
    out = _scaled_mm_nvfp4(nv, ca, sa_, one, cw, sw_, Sw, torch.bfloat16).double() * St.double()[:, None]
    da = nv.dequantize(ca, sa_, one).double() * St.double()[:, None]
    dw = nv.dequantize(cw, sw_, Sw).double()
    _check(out, da @ dw.T, da.abs() @ dw.abs().T)
