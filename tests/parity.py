"""GPU-vs-oracle comparison helpers (the parity metric).

A group matches when its scale byte and its 8 code bytes are equal.  At least
99.99% of groups must match; every mismatched group must have an exact
(oracle-evaluated) loss within 1e-6 relative of the oracle's own choice
(equal when that loss is 0).  h must agree within 1e-5 relative per column
(exactly 0 where the oracle's is 0).  Sweep parity feeds both sides the same
h bytes (the GPU's).
"""
from __future__ import annotations

import numpy as np
import torch

MATCH_FRACTION = 0.9999
LOSS_RTOL = 1e-6
H_RTOL = 1e-5


def to_bits(W: torch.Tensor) -> np.ndarray:
    return W.detach().cpu().contiguous().view(torch.uint16).numpy()


def check_h(h_gpu: np.ndarray, h_ref: np.ndarray):
    h_gpu = np.asarray(h_gpu, np.float64)
    h_ref = np.asarray(h_ref, np.float64)
    zero = h_ref == 0
    assert np.all(h_gpu[zero] == 0), "nonzero h where the oracle's is 0"
    rel = np.abs(h_gpu - h_ref) / np.where(zero, 1.0, np.abs(h_ref))
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= H_RTOL, f"h relative error {worst:.3e} > {H_RTOL}"
    return worst


def compare_groups(orc, w_bits: np.ndarray, h: np.ndarray | None, S: float,
                   gpu_codes: np.ndarray, gpu_scales: np.ndarray,
                   ref_codes: np.ndarray, ref_scales: np.ndarray) -> dict:
    """w_bits [n,16] u16, h [n,16] or None, codes [n,8], scales [n]."""
    n = w_bits.shape[0]
    gpu_codes = gpu_codes.reshape(n, 8)
    ref_codes = ref_codes.reshape(n, 8)
    gpu_scales = gpu_scales.reshape(n)
    ref_scales = ref_scales.reshape(n)
    match = (gpu_scales == ref_scales) & np.all(gpu_codes == ref_codes, axis=1)
    bad = np.flatnonzero(~match)
    res = {"groups": n, "mismatch": int(bad.size), "match_fraction": 1.0 - bad.size / max(n, 1),
           "worst_rel_loss": 0.0}
    if bad.size:
        hb = None if h is None else h.reshape(n, 16)[bad]
        lg = orc.packed_losses(w_bits[bad], hb, S, gpu_codes[bad], gpu_scales[bad])
        lr = orc.packed_losses(w_bits[bad], hb, S, ref_codes[bad], ref_scales[bad])
        rel = np.where(lr > 0, (lg - lr) / np.maximum(lr, 1e-300), np.where(lg > 0, np.inf, 0.0))
        res["worst_rel_loss"] = float(rel.max())
        res["bad_examples"] = [(int(i), int(gpu_scales[i]), int(ref_scales[i])) for i in bad[:5]]
    return res


def assert_parity(res: dict, what: str = ""):
    assert res["match_fraction"] >= MATCH_FRACTION, f"{what}: {res}"
    assert res["worst_rel_loss"] <= LOSS_RTOL, f"{what}: {res}"


def matrix_groups(bits: np.ndarray, codes: np.ndarray, scales: np.ndarray, h: np.ndarray | None):
    """Flatten a [rows, in] matrix and its outputs into per-group arrays."""
    rows, n = bits.shape
    G = n // 16
    w = bits.reshape(rows * G, 16)
    hh = None if h is None else np.broadcast_to(h.reshape(1, G, 16), (rows, G, 16)).reshape(-1, 16)
    return w, hh, codes.reshape(rows * G, 8), scales.reshape(rows * G)
