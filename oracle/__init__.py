"""CPU oracle for Hessian-weighted NVFP4 block-scale selection.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``block_scale_search_b200``) never imports it, and this package
never imports the product.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, fp64, exact decisions);
this module only builds it with gcc, loads it with ctypes and marshals numpy
arrays.  ``parallel_*`` helpers split rows / columns across host threads; the
C functions stay single-threaded (ctypes releases the GIL during each call).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "libnvfp4_oracle.so")
_lock = threading.Lock()
_lib = None

# gcc flags: IEEE float semantics, no contraction into FMAs, no fast-math.
CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library in-tree (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "nvfp4_oracle.h"))
    ):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(_LIB)
            u16p, f32p, u8p, i8p, f64p = (C.POINTER(t) for t in
                                          (C.c_uint16, C.c_float, C.c_uint8, C.c_int8, C.c_double))
            i64 = C.c_int64
            L.orc_e4m3_value.argtypes = [C.c_int]
            L.orc_e4m3_value.restype = C.c_double
            L.orc_e4m3_nearest.argtypes = [C.c_double]
            L.orc_e4m3_nearest.restype = C.c_int
            L.orc_e2m1_index.argtypes = [C.c_double, C.c_double]
            L.orc_e2m1_index.restype = C.c_int
            L.orc_group_loss.argtypes = [u16p, f32p, C.c_float, C.c_int]
            L.orc_group_loss.restype = C.c_double
            L.orc_diag_hessian.argtypes = [u16p, i64, i64, i64, f32p, C.c_int]
            L.orc_diag_hessian.restype = None
            L.orc_global_scale.argtypes = [u16p, i64, i64, i64, C.c_float, f32p, f32p]
            L.orc_global_scale.restype = C.c_int
            L.orc_base_code.argtypes = [u16p, C.c_float]
            L.orc_base_code.restype = C.c_int
            L.orc_sweep_group.argtypes = [u16p, f32p, C.c_float, C.c_int, C.c_int, u8p, u8p, i8p, f64p]
            L.orc_sweep_group.restype = None
            L.orc_sweep_quantize.argtypes = [u16p, i64, i64, i64, f32p, C.c_float, C.c_int, C.c_int,
                                             u8p, u8p, i8p]
            L.orc_sweep_quantize.restype = None
            L.orc_sweep_group_list.argtypes = [u16p, f32p, i64, C.c_float, C.c_int, C.c_int,
                                               u8p, u8p, i8p, f64p]
            L.orc_sweep_group_list.restype = None
            L.orc_group_loss_list.argtypes = [u16p, f32p, i64, C.c_float, u8p, f64p]
            L.orc_group_loss_list.restype = None
            L.orc_packed_loss_list.argtypes = [u16p, f32p, i64, C.c_float, u8p, u8p, f64p]
            L.orc_packed_loss_list.restype = None
            L.orc_quantize_activations.argtypes = [u16p, i64, i64, i64, C.c_float, C.c_int,
                                                   C.c_int, f32p, u8p, u8p, i8p]
            L.orc_quantize_activations.restype = C.c_int
            L.orc_dequantize.argtypes = [u8p, u8p, C.c_float, i64, i64, f32p]
            L.orc_dequantize.restype = None
            L.orc_sweep_group_f32_list.argtypes = [f32p, f32p, i64, C.c_float, C.c_int, C.c_int,
                                                   u8p, u8p, i8p, f64p]
            L.orc_sweep_group_f32_list.restype = None
            L.orc_group_loss_f32.argtypes = [f32p, f32p, C.c_float, C.c_int]
            L.orc_group_loss_f32.restype = C.c_double
            L.orc_base_code_f32.argtypes = [f32p, C.c_float]
            L.orc_base_code_f32.restype = C.c_int
            L.orc_e2m1_quantize_list.argtypes = [f32p, f64p, i64, u8p]
            L.orc_e2m1_quantize_list.restype = None
            _lib = L
    return _lib


# ---------------------------------------------------------------- marshalling

def _p(a: np.ndarray, ct):
    return a.ctypes.data_as(C.POINTER(ct))


def _bf16_bits(a) -> np.ndarray:
    """Accept a uint16 array of bf16 bit patterns or a torch bf16 tensor."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch  # local: only for the view
        return a.detach().cpu().contiguous().view(torch.uint16).numpy()
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _h_arr(h):
    if h is None:
        return None
    if hasattr(h, "detach"):
        h = h.detach().cpu().numpy()
    return np.ascontiguousarray(h, dtype=np.float32)


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(int(code))


def e4m3_nearest(f: float) -> int:
    return lib().orc_e4m3_nearest(float(f))


def e2m1_index(a: float, vS: float) -> int:
    return lib().orc_e2m1_index(float(a), float(vS))


def e4m3_table() -> np.ndarray:
    return np.array([e4m3_value(c) for c in range(127)], dtype=np.float64)


def group_loss(w16, h16, S: float, code: int) -> float:
    w = _bf16_bits(w16).reshape(16)
    h = _h_arr(h16)
    return lib().orc_group_loss(_p(w, C.c_uint16), None if h is None else _p(h, C.c_float),
                                float(S), int(code))


def base_code(w16, S: float) -> int:
    w = _bf16_bits(w16).reshape(16)
    return lib().orc_base_code(_p(w, C.c_uint16), float(S))


def diag_hessian(X, h=None, accumulate=False) -> np.ndarray:
    X = _bf16_bits(X)
    T, n = X.shape
    out = np.zeros(n, np.float32) if h is None else np.array(h, dtype=np.float32, copy=True)
    lib().orc_diag_hessian(_p(X, C.c_uint16), T, n, n, _p(out, C.c_float), int(bool(accumulate)))
    return out


def global_scale(W, q_max: float = 448.0):
    """Returns (S, amax, status)."""
    W = _bf16_bits(W)
    o, n = W.shape
    S = np.zeros(1, np.float32)
    am = np.zeros(1, np.float32)
    st = lib().orc_global_scale(_p(W, C.c_uint16), o, n, n, float(q_max), _p(S, C.c_float),
                                _p(am, C.c_float))
    return np.float32(S[0]), np.float32(am[0]), st


def sweep_quantize(W, h, S: float, lo: int, hi: int):
    """Single-threaded whole-matrix sweep: (codes[out,in/2], scales[out,in/16], offsets)."""
    W = _bf16_bits(W)
    o, n = W.shape
    h = _h_arr(h)
    codes = np.zeros((o, n // 2), np.uint8)
    scales = np.zeros((o, n // 16), np.uint8)
    offs = np.zeros((o, n // 16), np.int8)
    lib().orc_sweep_quantize(_p(W, C.c_uint16), o, n, n, None if h is None else _p(h, C.c_float),
                             float(S), int(lo), int(hi), _p(codes, C.c_uint8), _p(scales, C.c_uint8),
                             _p(offs, C.c_int8))
    return codes, scales, offs


def sweep_groups(w, h, S: float, lo: int, hi: int):
    """n independent groups: w[n,16] bf16 bits, h[n,16] or None.
    Returns (codes[n,8], scales[n], offsets[n], losses[n])."""
    w = _bf16_bits(w).reshape(-1, 16)
    n = w.shape[0]
    h = _h_arr(h)
    if h is not None:
        h = h.reshape(n, 16)
    codes = np.zeros((n, 8), np.uint8)
    scales = np.zeros(n, np.uint8)
    offs = np.zeros(n, np.int8)
    loss = np.zeros(n, np.float64)
    lib().orc_sweep_group_list(_p(w, C.c_uint16), None if h is None else _p(h, C.c_float), n,
                               float(S), int(lo), int(hi), _p(codes, C.c_uint8),
                               _p(scales, C.c_uint8), _p(offs, C.c_int8), _p(loss, C.c_double))
    return codes, scales, offs, loss


def group_losses(w, h, S: float, codes) -> np.ndarray:
    """Exact-evaluator loss of n groups at the given scale codes."""
    w = _bf16_bits(w).reshape(-1, 16)
    n = w.shape[0]
    h = _h_arr(h)
    if h is not None:
        h = h.reshape(n, 16)
    c = np.ascontiguousarray(codes, dtype=np.uint8).reshape(n)
    out = np.zeros(n, np.float64)
    lib().orc_group_loss_list(_p(w, C.c_uint16), None if h is None else _p(h, C.c_float), n,
                              float(S), _p(c, C.c_uint8), _p(out, C.c_double))
    return out


def packed_losses(w, h, S: float, codes, scales) -> np.ndarray:
    """Exact weighted loss of groups as packed by any quantizer: w[n,16] bf16
    bits, h[n,16] or None, codes[n,8], scales[n]."""
    w = _bf16_bits(w).reshape(-1, 16)
    n = w.shape[0]
    h = _h_arr(h)
    if h is not None:
        h = h.reshape(n, 16)
    cd = np.ascontiguousarray(codes, dtype=np.uint8).reshape(n, 8)
    sc = np.ascontiguousarray(scales, dtype=np.uint8).reshape(n)
    out = np.zeros(n, np.float64)
    lib().orc_packed_loss_list(_p(w, C.c_uint16), None if h is None else _p(h, C.c_float), n,
                               float(S), _p(cd, C.c_uint8), _p(sc, C.c_uint8), _p(out, C.c_double))
    return out


def quantize_activations(A, q_max: float = 256.0, lo: int = -3, hi: int = 7):
    """Per-token online quantization of A[tokens, in] (bf16 bits or torch bf16).
    Returns (S[tokens] float32, codes[tokens,in/2], scales[tokens,in/16],
    offsets[tokens,in/16], status)."""
    A = _bf16_bits(A)
    t, n = A.shape
    S = np.zeros(t, np.float32)
    codes = np.zeros((t, n // 2), np.uint8)
    scales = np.zeros((t, n // 16), np.uint8)
    offs = np.zeros((t, n // 16), np.int8)
    st = lib().orc_quantize_activations(_p(A, C.c_uint16), t, n, n, float(q_max), int(lo), int(hi),
                                        _p(S, C.c_float), _p(codes, C.c_uint8),
                                        _p(scales, C.c_uint8), _p(offs, C.c_int8))
    return S, codes, scales, offs, st


def dequantize(codes, scales, S: float) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    o, half = codes.shape
    out = np.zeros((o, half * 2), np.float32)
    lib().orc_dequantize(_p(codes, C.c_uint8), _p(scales, C.c_uint8), float(S), o, half * 2,
                         _p(out, C.c_float))
    return out


def sweep_group_f32_list(w, h, S: float, lo: int, hi: int):
    """The windowed sweep of n FP32 groups w[n,16] (h[n,16] or None): (codes
    [n,8], scales [n], offsets [n], losses [n])."""
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1, 16)
    n = w.shape[0]
    h = None if h is None else np.ascontiguousarray(h, dtype=np.float32).reshape(n, 16)
    codes = np.zeros((n, 8), np.uint8)
    scales = np.zeros(n, np.uint8)
    offs = np.zeros(n, np.int8)
    loss = np.zeros(n, np.float64)
    lib().orc_sweep_group_f32_list(_p(w, C.c_float), None if h is None else _p(h, C.c_float), n,
                                   float(S), int(lo), int(hi), _p(codes, C.c_uint8),
                                   _p(scales, C.c_uint8), _p(offs, C.c_int8),
                                   _p(loss, C.c_double))
    return codes, scales, offs, loss


def group_loss_f32(w, h, S: float, code: int) -> float:
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(16)
    hp = None if h is None else _p(np.ascontiguousarray(h, dtype=np.float32).reshape(16), C.c_float)
    return lib().orc_group_loss_f32(_p(w, C.c_float), hp, float(S), int(code))


def e2m1_quantize_list(w, vS) -> np.ndarray:
    """Nibbles of FP32 values w[n] at their own exact scales vS[n] (0: nibble 0)."""
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    vS = np.ascontiguousarray(vS, dtype=np.float64).reshape(-1)
    nib = np.zeros(w.size, np.uint8)
    lib().orc_e2m1_quantize_list(_p(w, C.c_float), _p(vS, C.c_double), w.size, _p(nib, C.c_uint8))
    return nib


# ---------------------------------------------------------- threaded drivers

def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def parallel_sweep_quantize(W, h, S: float, lo: int, hi: int, threads: int | None = None):
    """Row-chunked multi-threaded driver around the single-threaded C sweep."""
    W = _bf16_bits(W)
    o, n = W.shape
    h = _h_arr(h)
    codes = np.zeros((o, n // 2), np.uint8)
    scales = np.zeros((o, n // 16), np.uint8)
    offs = np.zeros((o, n // 16), np.int8)
    threads = threads or default_threads()
    L = lib()
    hp = None if h is None else _p(h, C.c_float)

    def run(r0, r1):
        L.orc_sweep_quantize(_p(W[r0:r1], C.c_uint16), r1 - r0, n, n, hp, float(S), int(lo),
                             int(hi), _p(codes[r0:r1], C.c_uint8), _p(scales[r0:r1], C.c_uint8),
                             _p(offs[r0:r1], C.c_int8))

    step = max(1, -(-o // (threads * 4)))
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda r: run(r, min(o, r + step)), range(0, o, step)))
    return codes, scales, offs


def parallel_quantize_activations(A, q_max: float = 256.0, lo: int = -3, hi: int = 7,
                                  threads: int | None = None):
    """Token-chunked multi-threaded driver around orc_quantize_activations;
    same returns as quantize_activations."""
    A = _bf16_bits(A)
    t, n = A.shape
    S = np.zeros(t, np.float32)
    codes = np.zeros((t, n // 2), np.uint8)
    scales = np.zeros((t, n // 16), np.uint8)
    offs = np.zeros((t, n // 16), np.int8)
    threads = threads or default_threads()
    L = lib()

    def run(r0, r1):
        return L.orc_quantize_activations(_p(A[r0:r1], C.c_uint16), r1 - r0, n, n, float(q_max),
                                          int(lo), int(hi), _p(S[r0:r1], C.c_float),
                                          _p(codes[r0:r1], C.c_uint8), _p(scales[r0:r1], C.c_uint8),
                                          _p(offs[r0:r1], C.c_int8))

    step = max(1, -(-t // (threads * 4)))
    with ThreadPoolExecutor(threads) as ex:
        rcs = list(ex.map(lambda r: run(r, min(t, r + step)), range(0, t, step)))
    return S, codes, scales, offs, (min(rcs) if rcs else 0)


def parallel_diag_hessian(X, threads: int | None = None) -> np.ndarray:
    """Column-chunked multi-threaded driver around the C diag-Hessian."""
    X = _bf16_bits(X)
    T, n = X.shape
    out = np.zeros(n, np.float32)
    threads = threads or default_threads()
    L = lib()
    step = max(1, -(-n // threads))

    def run(c0):
        c1 = min(n, c0 + step)
        L.orc_diag_hessian(_p(X[:, c0:], C.c_uint16), T, c1 - c0, n, _p(out[c0:c1], C.c_float), 0)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(run, range(0, n, step)))
    return out
