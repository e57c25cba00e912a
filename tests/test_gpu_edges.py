"""Exhaustive decode and out-of-bounds write checks on a B200.

* every E4M3 scale code (0..126) with every packed byte (0..255), at a normal,
  a denormal and a zero global scale, decodes bit-exactly as the oracle does;
* every entry point writes only its outputs: each output is carved out of a
  larger buffer filled with a canary pattern, and the canary must survive."""
import numpy as np
import pytest
import torch

from parity import to_bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
CANARY = 0xA5


@pytest.fixture(scope="module")
def nv():
    import block_scale_search_b200 as nv
    nv.lib()
    return nv


@pytest.mark.parametrize("S", [0.0078125, 3.0e-42, 0.0, 1.7e4])
def test_dequantize_every_scale_and_byte(orc, nv, S):
    codes = np.tile(np.arange(256, dtype=np.uint8), (127, 1))        # [127, 256] -> 512 elements/row
    scales = np.repeat(np.arange(127, dtype=np.uint8)[:, None], 32, axis=1)
    Sd = torch.tensor([S], dtype=torch.float32, device=DEV)
    out = nv.dequantize(torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV), Sd)
    ref = orc.dequantize(codes, scales, float(np.float32(S)))
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def _carve(n_bytes, dtype, align=256, pad=4096):
    """A view of n_bytes inside a canary-filled buffer (pad bytes each side)."""
    buf = torch.full((pad + n_bytes + pad,), CANARY, dtype=torch.uint8, device=DEV)
    view = buf[pad:pad + n_bytes]
    assert view.data_ptr() % align == 0
    return buf, view.view(dtype)


def _canary_ok(buf, n_bytes, pad=4096):
    b = buf.cpu().numpy()
    return bool(np.all(b[:pad] == CANARY) and np.all(b[pad + n_bytes:] == CANARY))


@pytest.mark.parametrize("out,inp", [(1, 16), (7, 48), (33, 1040), (129, 2048)])
def test_no_write_outside_outputs(nv, out, inp):
    import workloads
    W = workloads.weight(out, inp, 0.02, 0.01, 10.0, 300 + inp, DEV)
    X = workloads.calib(45, inp, 1.0, 400 + inp, DEV)

    hb, h = _carve(inp * 4, torch.float32)
    ws = torch.empty(nv.nvfp4_diag_hessian_workspace_size(45, inp), dtype=torch.uint8, device=DEV)
    nv.nvfp4_diag_hessian(X, 45, inp, inp, h, 0, ws, ws.numel())
    Sb, S = _carve(4, torch.float32)
    Ab, A = _carve(4, torch.float32)
    Tb, T = _carve(4, torch.int32)
    gws = torch.empty(nv.nvfp4_global_scale_workspace_size(out, inp), dtype=torch.uint8, device=DEV)
    nv.nvfp4_global_scale(W, out, inp, inp, 448.0, S, A, T, gws, gws.numel())
    cb, codes = _carve(out * inp // 2, torch.uint8)
    sb, scales = _carve(out * inp // 16, torch.uint8)
    ob, offs = _carve(out * inp // 16, torch.int8)
    nv.nvfp4_scale_sweep_quantize(W, out, inp, inp, h, S, -9, 6, codes, scales, offs)
    db, deq = _carve(out * inp * 4, torch.float32)
    nv.nvfp4_dequantize(codes, scales, S, out, inp, deq)
    torch.cuda.synchronize()
    for buf, n in ((hb, inp * 4), (Sb, 4), (Ab, 4), (Tb, 4), (cb, out * inp // 2),
                   (sb, out * inp // 16), (ob, out * inp // 16), (db, out * inp * 4)):
        assert _canary_ok(buf, n)
    # and the outputs were all written (no canary left inside them)
    assert h.min().item() >= 0 and T.item() == 0
    sc = scales.cpu().numpy()
    assert np.all(sc <= 126)


def test_no_write_outside_grouped_outputs(nv):
    import workloads
    counts = [3, 0, 700, 11]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    X = workloads.calib(int(offs[-1]), 64, 1.0, 77, DEV)
    hb, h = _carve(4 * 64 * 4, torch.float32)
    h = h.view(4, 64)
    ws = torch.empty(nv.nvfp4_diag_hessian_grouped_workspace_size(int(offs[-1]), 4, 64),
                     dtype=torch.uint8, device=DEV)
    nv.nvfp4_diag_hessian_grouped(X, torch.from_numpy(offs).to(DEV), 4, int(offs[-1]), 64, 64, h,
                                  0, ws, ws.numel())
    torch.cuda.synchronize()
    assert _canary_ok(hb, 4 * 64 * 4)
    assert not h[1].any() and h[2].min().item() > 0
