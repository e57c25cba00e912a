"""Pins for the oracle's online activation quantization (ScaleSweep summary,
W+A settings: activations quantized to NVFP4 with the MSE sweep, window
[-3, +7], global scale S = max|x| / (256 * 6) taken per token).

Checked against closed forms, an exact power-of-two invariance, and brute
force over all 126 scale codes; no GPU needed."""
import numpy as np
import torch

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def bf16_bits(t):
    return t.to(torch.bfloat16).view(torch.uint16).numpy()


def _act_rows(tokens, n, seed):
    """Activation-like rows: Gaussian times lognormal channel scales, a few
    outlier channels, per-token magnitude spread."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(tokens, n, generator=g, dtype=torch.float64)
    x *= torch.exp(torch.randn(1, n, generator=g, dtype=torch.float64))
    x[:, :: max(1, n // 7)] *= 30.0
    x *= torch.exp(0.5 * torch.randn(tokens, 1, generator=g, dtype=torch.float64))
    return x


def test_power_of_two_row_scaling_is_exact(orc):
    """Scaling a token by 2^k scales its S by exactly 2^k and leaves every code,
    scale byte and offset unchanged (all FP32 steps scale exactly away from
    underflow and overflow).  A row given another row's S, or the tensor's,
    would shift its scale bytes."""
    base = _act_rows(1, 512, 7)
    ks = np.array([0, 9, -13, 27, -30, 4, 1, -1])
    A = torch.cat([base * 2.0 ** int(k) for k in ks])
    S, codes, scales, offs, st = orc.quantize_activations(bf16_bits(A), 256.0, -3, 7)
    assert st == 0
    for t, k in enumerate(ks):
        assert S[t] == np.float32(S[0] * np.float32(2.0 ** int(k)))
        np.testing.assert_array_equal(codes[t], codes[0])
        np.testing.assert_array_equal(scales[t], scales[0])
        np.testing.assert_array_equal(offs[t], offs[0])
    assert len(set(S.tolist())) == len(ks)


def test_closed_form_scale_and_code(orc):
    """amax 1536 with Q = 256, and amax 2688 with Q = 448, give S = 1 exactly.
    A group holding 1536 and zeros then has base code 120 (value 256): 1536/256
    = 6 reconstructs exactly, every smaller code saturates below 1536, so code
    120 wins at offset 0 and element 0 packs as nibble 7."""
    A = torch.zeros(2, 32, dtype=torch.float64)
    A[0, 0] = 1536.0
    A[0, 17] = -3.0
    A[1, 0] = 2688.0
    S, codes, scales, offs, st = orc.quantize_activations(bf16_bits(A), 256.0, -3, 7)
    assert st == 0 and S[0] == 1.0
    assert scales[0, 0] == 120 and offs[0, 0] == 0 and codes[0, 0] == 0x07
    assert not codes[0, 1:8].any()
    S2, _, _, _, _ = orc.quantize_activations(bf16_bits(A[1:]), 448.0, -3, 7)
    assert S2[0] == 1.0
    # group 1 of row 0: a = 3, base = nearest(0.5) = code 48 (v = 0.5), 3 / 0.5 = 6;
    # element 17 is odd, so its nibble (sign | 7) sits in the high half of byte 8
    assert scales[0, 1] == 48 and codes[0, 8] == 0xF0


def test_zero_and_nonfinite_rows(orc):
    A = _act_rows(5, 64, 11)
    A[1] = 0.0
    A[2, 5] = float("inf")
    A[3, 60] = float("nan")
    bits = bf16_bits(A)
    S, codes, scales, offs, st = orc.quantize_activations(bits, 256.0, -3, 7)
    assert st == -5
    assert S[1] == 0.0 and np.isnan(S[2]) and np.isnan(S[3])
    for t in (1, 2, 3):
        assert not codes[t].any() and not scales[t].any() and not offs[t].any()
    for t in (0, 4):   # the other rows are exactly what they are alone
        S1, c1, s1, o1, st1 = orc.quantize_activations(bits[t:t + 1], 256.0, -3, 7)
        assert st1 == 0 and S1[0] == S[t]
        np.testing.assert_array_equal(c1[0], codes[t])
        np.testing.assert_array_equal(s1[0], scales[t])


def test_rows_follow_their_tokens(orc):
    """Permuting the tokens permutes every output the same way."""
    A = bf16_bits(_act_rows(9, 128, 13))
    perm = np.array([4, 0, 8, 2, 7, 1, 6, 3, 5])
    ref = orc.quantize_activations(A, 256.0, -3, 7)
    got = orc.quantize_activations(np.ascontiguousarray(A[perm]), 256.0, -3, 7)
    for r, g in zip(ref[:4], got[:4]):
        np.testing.assert_array_equal(r[perm], g)


def test_window_reaches_the_full_mse_optimum(orc):
    """ScaleSweep Lemma 4.1 / 4.3 with each token's own S: for groups whose base
    code is normal, the best loss in [-3, +7] equals the best over all 126
    codes (brute force with the exact group loss)."""
    A = bf16_bits(_act_rows(8, 256, 17))
    S, codes, scales, offs, st = orc.quantize_activations(A, 256.0, -3, 7)
    assert st == 0
    checked = 0
    for t in range(A.shape[0]):
        w = A[t].reshape(-1, 16)
        n = w.shape[0]
        full = np.min(np.stack([orc.group_losses(w, None, S[t], np.full(n, c, np.uint8))
                                for c in range(1, 127)]), axis=0)
        got = orc.group_losses(w, None, S[t], scales[t])
        base = np.array([orc.base_code(w[i], S[t]) for i in range(n)])
        sel = base >= 8
        checked += int(sel.sum())
        np.testing.assert_array_equal(got[sel], full[sel])
        assert np.all(got >= full)
    assert checked > 64
