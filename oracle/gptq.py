"""CPU oracle of H-Scale as the local quantizer inside GPTQ (TEST
INFRASTRUCTURE ONLY, like the rest of this package).

H-Scale summary, sec. B "Implementation" and "GPTQ Integration": in GPTQ,
H-Scale replaces only the local quantization call; the inverse-Cholesky
processing, the error computation and its propagation stay GPTQ's own.  The
GPTQ steps are the standard algorithm (column order as given, no reordering):

  * H = X^T X (the calibration Gram matrix) in FP64; a column whose diagonal is
    0 gets H_jj = 1 and zero weights; H += damp * mean(diag H) * I;
  * U = the upper Cholesky factor of H^-1 (H^-1 = U^T U);
  * for each column j in order: quantize w_j, err = (w_j - q_j) / U_jj, and
    w_k -= err * U_jk for every later column k.

The local call (readings, stated where the page is silent):
  * at the first column of each 16-column group, every row's E4M3 scale code
    for that group is chosen by the H-Scale windowed sweep on the group's
    current (error-updated) weights, rounded to FP32 -- the precision a
    quantizer sees -- with h = diag(X^T X) as the standalone path computes it
    and the global scale S of the original weights;
  * each column of the group is then quantized at its turn, with that scale:
    the exact E2M1 round-to-nearest-even of its FP32 current value; its error
    is taken on the FP64 current value.

Everything is FP64 numpy (matmul, inverse and Cholesky are library routines
used as steps); the per-group sweep and the E2M1 decisions are the C oracle's.
"""
from __future__ import annotations

import numpy as np

from . import _bf16_bits, diag_hessian, e2m1_quantize_list, e4m3_value, global_scale
from . import sweep_group_f32_list

_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_V = np.array([max(e4m3_value(c), 0.0) for c in range(127)], dtype=np.float64)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def inverse_cholesky_upper(X_bits: np.ndarray, damp: float = 0.01):
    """(U, dead): U upper with U^T U = (X^T X + damp mean(diag) I)^-1 after the
    dead-column rule; dead marks the columns whose diagonal was 0."""
    Xf = bf16_to_f64(_bf16_bits(X_bits))
    H = Xf.T @ Xf
    dead = np.diag(H) == 0.0
    H[dead, dead] = 1.0
    H += damp * np.mean(np.diag(H)) * np.eye(H.shape[0])
    Hinv = np.linalg.inv(H)
    U = np.linalg.cholesky(Hinv).T
    return U, dead, H


def decode(nib: np.ndarray, scale: np.ndarray, S: float) -> np.ndarray:
    """FP64 value of nibbles at E4M3 scale codes (codes 0: value 0)."""
    mag = _GRID[nib & 7] * _V[scale] * np.float64(S)
    return np.where(nib & 8, -mag, mag)


def gptq_hscale(W, X, q_max: float = 448.0, lo: int = -9, hi: int = 6, damp: float = 0.01,
                weighted: bool = True, trace=None, S=None):
    """GPTQ with the H-Scale local call.  W: bf16 [out, in] (bits or torch);
    X: bf16 [tokens, in].  Returns (codes [out, in/2], scales [out, in/16], S,
    Q [out, in] the FP64 dequantized weights, h [in]).  trace(j, W, Q) is called
    after column j's error has been propagated, with the current FP64 weights
    and the columns quantized so far.  S, if given, is the global scale to use
    instead of W's own: rows are independent in GPTQ given H, so some rows of a
    larger matrix run alone with that matrix's S give that matrix's rows."""
    Wb = _bf16_bits(W)
    Xb = _bf16_bits(X)
    out, n = Wb.shape
    assert n % 16 == 0 and Xb.shape[1] == n
    if S is None:
        S, _amax, st = global_scale(Wb, q_max)
        if st != 0:
            raise ValueError("non-finite weights")
    S = np.float32(S)
    h = diag_hessian(Xb)
    U, dead, _H = inverse_cholesky_upper(Xb, damp)
    Wc = bf16_to_f64(Wb)
    Wc[:, dead] = 0.0
    nib = np.zeros((out, n), np.uint8)
    scales = np.zeros((out, n // 16), np.uint8)
    Q = np.zeros((out, n), np.float64)
    for g in range(n // 16):
        c0 = 16 * g
        wg = Wc[:, c0:c0 + 16].astype(np.float32)
        hg = np.broadcast_to(h[c0:c0 + 16], (out, 16)) if weighted else None
        _, sc, _, _ = sweep_group_f32_list(wg, hg, float(S), lo, hi)
        scales[:, g] = sc
        vS = _V[sc] * np.float64(S)                    # exact: E4M3 x FP32
        for i in range(16):
            j = c0 + i
            w = Wc[:, j]
            nj = e2m1_quantize_list(w.astype(np.float32), vS)
            q = decode(nj, sc, S)
            nib[:, j] = nj
            Q[:, j] = q
            err = (w - q) / U[j, j]
            Wc[:, j + 1:] -= np.outer(err, U[j, j + 1:])
            if trace is not None:
                trace(j, Wc, Q)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return codes, scales, np.float32(S), Q, h
