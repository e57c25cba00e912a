"""Pins of the GPTQ oracle with the H-Scale local call (H-Scale summary, sec. B
"GPTQ Integration"): each checks it against something other than itself --
the standalone sweep where GPTQ has nothing to propagate, the bf16 oracle on
values both can hold, the damped least-squares re-fit that GPTQ's update is,
and the expected gain on correlated inputs."""
import numpy as np
import pytest

import oracle
from oracle import gptq


def _w(out, n, seed, frac=0.01):
    import workloads
    return workloads.weight(out, n, 0.02, frac, 10.0, seed)


def test_uncorrelated_inputs_reduce_to_the_sweep():
    """X = 2 I: H = 4 I, U is diagonal, nothing propagates, and GPTQ with the
    local call is the standalone windowed sweep with h = 4."""
    import torch
    n = 256
    W = _w(96, n, 1)
    X = (2.0 * torch.eye(n)).to(torch.bfloat16)
    codes, scales, S, _, h = gptq.gptq_hscale(W, X, lo=-9, hi=6)
    assert np.all(h == 4.0)
    rc, rs, _ = oracle.sweep_quantize(W, h, float(S), -9, 6)
    np.testing.assert_array_equal(scales, rs)
    np.testing.assert_array_equal(codes, rc)


@pytest.mark.parametrize("weighted", [False, True])
def test_fp32_local_call_equals_the_bf16_sweep_on_bf16_values(weighted):
    rng = np.random.default_rng(3)
    W = _w(200, 512, 4, frac=0.02)
    bits = oracle._bf16_bits(W).reshape(-1, 16)
    bits[5] = 0                                     # an all-zero group
    bits[6, :8] = 0x8000                            # negative zeros
    h = rng.lognormal(0.0, 1.5, size=bits.shape).astype(np.float32) if weighted else None
    S = float(oracle.global_scale(bits.reshape(200, 512), 448.0)[0])
    rc, rs, ro, rl = oracle.sweep_groups(bits, h, S, -9, 6)
    f = gptq.bf16_to_f64(bits).astype(np.float32)
    fc, fs, fo, fl = oracle.sweep_group_f32_list(f, h, S, -9, 6)
    np.testing.assert_array_equal(fc, rc)
    np.testing.assert_array_equal(fs, rs)
    np.testing.assert_array_equal(fo, ro)
    np.testing.assert_array_equal(fl, rl)


def test_propagation_is_the_damped_least_squares_refit():
    """After column j, GPTQ's remaining columns minimise the damped output
    error with the quantized columns held fixed: V = W_> + A H_<> H_>>^-1,
    A = W_<= - Q_<=, computed here by a linear solve on the damped H (no
    Cholesky, no inverse)."""
    import torch
    import workloads
    n = 64
    W = _w(12, n, 7)
    Z = workloads.calib(200, n, 1.0, 8).float()
    X = (Z @ (torch.eye(n) + 0.3 * torch.randn(n, n, generator=torch.Generator().manual_seed(9)))
         ).to(torch.bfloat16)
    _, _, Hd = gptq.inverse_cholesky_upper(oracle._bf16_bits(X))
    W0 = gptq.bf16_to_f64(oracle._bf16_bits(W))
    seen = []

    def trace(j, Wc, Q):
        if j in (0, 5, 15, 16, 40, 62):
            A = W0[:, :j + 1] - Q[:, :j + 1]
            V = W0[:, j + 1:] + np.linalg.solve(Hd[j + 1:, j + 1:], (A @ Hd[:j + 1, j + 1:]).T).T
            np.testing.assert_allclose(Wc[:, j + 1:], V, rtol=1e-9, atol=1e-12)
            seen.append(j)

    gptq.gptq_hscale(W, X, trace=trace)
    assert seen == [0, 5, 15, 16, 40, 62]


@pytest.mark.parametrize("seed", [11, 12, 13])
def test_correlated_inputs_lower_the_output_error(seed):
    """On inputs with correlated channels GPTQ's propagation lowers the layer
    output error below the standalone sweep's (the reason to combine them)."""
    import torch
    import workloads
    n = 128
    W = _w(64, n, seed)
    Z = workloads.calib(512, n, 1.0, seed + 100).float()
    mix = torch.eye(n) + 0.5 * torch.randn(n, n, generator=torch.Generator().manual_seed(seed))
    X = (Z @ mix).to(torch.bfloat16)
    codes, scales, S, Q, h = gptq.gptq_hscale(W, X)
    rc, rs, _ = oracle.sweep_quantize(W, h, float(S), -9, 6)
    nib = np.stack([rc & 15, rc >> 4], -1).reshape(64, n)
    Qr = gptq.decode(nib, np.repeat(rs, 16, 1), float(S))
    Wf = gptq.bf16_to_f64(oracle._bf16_bits(W))
    Xf = gptq.bf16_to_f64(oracle._bf16_bits(X))
    e_gptq = np.sum((Xf @ (Wf - Q).T) ** 2)
    e_sweep = np.sum((Xf @ (Wf - Qr).T) ** 2)
    assert e_gptq < 0.95 * e_sweep, (e_gptq, e_sweep)
    # what the codes decode to is what GPTQ reconstructed
    qn = np.stack([codes & 15, codes >> 4], -1).reshape(64, n)
    np.testing.assert_array_equal(gptq.decode(qn, np.repeat(scales, 16, 1), float(S)), Q)


def test_dead_columns_quantize_to_zero():
    import workloads
    n = 64
    W = _w(32, n, 21)
    X = workloads.calib(100, n, 1.0, 22)
    X[:, 17] = 0
    X[:, 40:48] = 0
    codes, scales, S, Q, h = gptq.gptq_hscale(W, X)
    assert np.all(Q[:, 17] == 0) and np.all(Q[:, 40:48] == 0)
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(32, n)
    assert np.all(nib[:, 17] == 0) and np.all(nib[:, 40:48] == 0)


def _r_form(W, X, lo=-9, hi=6, damp=0.01, part=128, parts=4):
    """GPTQ restated in the form the device runs, FP64, no inverse of H: H =
    R R^T with R upper (R = J L J, L the lower Cholesky factor of J H J, J the
    order reversal); since W - Q = Err U with U = R^-1, a group's current
    weights are W_grp + (D[:, <g0] R[<g0, grp]) R_grp^-1 with D = W - Q; the
    later columns' sums P are brought up to date in lazy batches of `parts`
    parts of `part` columns (after each part for the next one, after each
    batch for all later columns)."""
    from oracle import e2m1_quantize_list, sweep_group_f32_list
    Wb, Xb = oracle._bf16_bits(W), oracle._bf16_bits(X)
    out, n = Wb.shape
    S, _, _ = oracle.global_scale(Wb, 448.0)
    h = oracle.diag_hessian(Xb)
    Xf = gptq.bf16_to_f64(Xb)
    H = Xf.T @ Xf
    dead = np.diag(H) == 0.0
    H[dead, dead] = 1.0
    H += damp * np.mean(np.diag(H)) * np.eye(n)
    J = np.eye(n)[::-1]
    R = J @ np.linalg.cholesky(J @ H @ J) @ J
    W0 = gptq.bf16_to_f64(Wb)
    W0[:, dead] = 0.0
    P, D = np.zeros((out, n)), np.zeros((out, n))
    nib = np.zeros((out, n), np.uint8)
    scales = np.zeros((out, n // 16), np.uint8)
    for j0 in range(0, n, part * parts):
        jend = min(j0 + part * parts, n)
        for c0 in range(j0, jend, part):
            c1 = min(c0 + part, jend)
            for g0 in range(c0, c1, 16):
                gs = slice(g0, g0 + 16)
                Ug = np.linalg.inv(R[gs, gs])
                w = W0[:, gs] + (P[:, gs] + D[:, c0:g0] @ R[c0:g0, gs]) @ Ug
                _, sc, _, _ = sweep_group_f32_list(
                    w.astype(np.float32), np.broadcast_to(h[gs], (out, 16)), float(S), lo, hi)
                scales[:, g0 // 16] = sc
                vS = gptq._V[sc] * np.float64(S)
                for i in range(16):
                    j = g0 + i
                    nib[:, j] = e2m1_quantize_list(w[:, i].astype(np.float32), vS)
                    q = gptq.decode(nib[:, j], sc, S)
                    w[:, i + 1:] -= np.outer((w[:, i] - q) * R[j, j], Ug[i, i + 1:])
                    D[:, j] = W0[:, j] - q
            if c1 < jend:
                P[:, c1:c1 + part] += D[:, j0:c1] @ R[j0:c1, c1:c1 + part]
        if jend < n:
            P[:, jend:] += D[:, j0:jend] @ R[j0:jend, jend:]
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8), scales


@pytest.mark.parametrize("n", [272, 400, 656])
def test_the_devices_r_form_gives_the_oracles_bytes(n):
    """The rearrangement the device runs (no inverse, lazy batches of 512 in
    parts of 128; here parts of 32 so that small widths cross several parts
    and batches) takes the same decisions as the oracle's U form in FP64: the
    two differ only in rounding order."""
    import torch
    rng = np.random.default_rng(n)
    W = _w(24, n, 50 + n)
    base = rng.normal(size=(768, 8)) @ rng.normal(size=(8, n))
    X = torch.from_numpy(base + 0.3 * rng.normal(size=(768, n)) * np.exp(rng.normal(size=n)))
    X = X.to(torch.bfloat16)
    oc, os_, *_ = gptq.gptq_hscale(W, X)
    rc, rs = _r_form(W, X, part=32, parts=4)
    np.testing.assert_array_equal(rs, os_)
    np.testing.assert_array_equal(rc, oc)


# --- direct pins of the FP32 forms the GPTQ oracle uses ----------------------

_GRID = [0, 1, 2, 3, 4, 6, 8, 12]   # E2M1 magnitudes times 2 (exact integers)


def _nearest_e2m1(a, vS):
    """Index of the E2M1 magnitude nearest to a / vS, exact ties to the even
    index, by exact rational arithmetic (the E2M1 definition, brute force)."""
    from fractions import Fraction
    x = Fraction(a) / Fraction(vS) * 2
    best = min(range(8), key=lambda k: (abs(x - _GRID[k]), k & 1))
    return best


def test_e2m1_quantize_list_is_the_nearest_grid_value():
    """Nibbles of FP32 values at their own exact scales: the nearest E2M1 value
    by exact arithmetic, ties to the even code, saturating at 6, sign in bit 3
    except for a zero magnitude -- on random values and on exact midpoints."""
    rng = np.random.default_rng(11)
    v = np.array([oracle.e4m3_value(c) for c in rng.integers(1, 127, 600)])
    S = np.float32(2.0 ** -7)
    vS = v * np.float64(S)                                   # exact
    w = (rng.standard_normal(600) * 4 * vS).astype(np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.5])
    k = rng.integers(0, 8, 400)
    vm = vS[:400]
    wm = (mids[k] * vm * rng.choice([-1.0, 1.0], 400)).astype(np.float32)
    assert np.all(wm.astype(np.float64) == mids[k] * vm * np.sign(wm))   # exact midpoints
    W = np.concatenate([w, wm, np.float32([0.0, -0.0, 1e-30, -1e-30])])
    VS = np.concatenate([vS, vm, vS[:4]])
    got = oracle.e2m1_quantize_list(W, VS)
    for x, s, g in zip(W, VS, got):
        m = _nearest_e2m1(abs(float(x)), float(s))
        want = m | (8 if (x < 0 and m != 0) else 0)
        assert g == want, (float(x), float(s), int(g), want)


def test_fp32_base_code_is_the_e4m3_rounding_of_two_fp32_divisions():
    """A one-candidate window returns the base code: E4M3 round-to-nearest-even
    (torch's float8_e4m3fn cast, saturated at 448) of fl32(fl32(a/6)/S), a the
    group's largest magnitude, clamped to [1, 126]; 0 for a zero group."""
    import torch
    rng = np.random.default_rng(12)
    w = (rng.standard_normal((500, 16)) * np.exp(rng.normal(0, 3, (500, 1)))).astype(np.float32)
    w[7] = 0.0
    S = np.float32(0.01)
    _, scales, _, _ = oracle.sweep_group_f32_list(w, None, float(S), 0, 0)
    a = np.abs(w).max(axis=1).astype(np.float32)
    t = (a / np.float32(6.0)).astype(np.float32) / S
    t = np.minimum(t.astype(np.float32), np.float32(448.0))
    code = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(int)
    want = np.where(a > 0, np.clip(code, 1, 126), 0)
    np.testing.assert_array_equal(scales.astype(int), want)


def test_fp32_group_loss_is_the_exact_weighted_error():
    """orc_group_loss_f32 against the weighted squared error computed in exact
    rational arithmetic from the brute-force nearest grid values (FP64 sums of
    exact terms: agreement to 1e-13)."""
    from fractions import Fraction
    rng = np.random.default_rng(13)
    S = np.float32(3e-4)
    for _ in range(40):
        w = (rng.standard_normal(16) * 0.02).astype(np.float32)
        h = rng.lognormal(0.0, 1.0, 16).astype(np.float32)
        code = int(rng.integers(40, 110))
        vS = oracle.e4m3_value(code) * float(S)
        exact = Fraction(0)
        for x, hx in zip(w, h):
            k = _nearest_e2m1(abs(float(x)), vS)
            e = Fraction(abs(float(x))) - Fraction(_GRID[k], 2) * Fraction(vS)
            exact += Fraction(float(hx)) * e * e
        got = oracle.group_loss_f32(w, h, float(S), code)
        assert abs(got - float(exact)) <= 1e-13 * float(exact), (got, float(exact))
