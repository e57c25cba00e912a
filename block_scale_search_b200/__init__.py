"""Python binding of libnvfp4hs (Hessian-weighted NVFP4 block-scale selection).

Argument marshalling only: every step runs in the CUDA kernels behind the C
ABI declared in ``include/nvfp4hs.h``.  PyTorch provides device memory and the
current stream.  The ``nvfp4_*`` functions mirror the C entry points one to
one; the lower-case helpers below them allocate outputs and workspaces with
torch and call those entry points.  There is no CPU fallback: if the shared
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

from . import _build

__all__ = [
    "NVFP4Error", "lib", "nvfp4_version", "nvfp4_diag_hessian_workspace_size",
    "nvfp4_diag_hessian", "nvfp4_global_scale_workspace_size", "nvfp4_global_scale",
    "nvfp4_global_scale_noalloc", "nvfp4_diag_hessian_grouped_workspace_size",
    "nvfp4_diag_hessian_grouped", "nvfp4_global_scale_batched_workspace_size",
    "nvfp4_global_scale_batched", "nvfp4_scale_sweep_quantize_batched_workspace_size",
    "nvfp4_scale_sweep_quantize_batched", "MatrixDesc", "SweepDesc",
    "nvfp4_scale_sweep_quantize_full", "scale_sweep_quantize_full", "nvfp4_debug_row_counters",
    "nvfp4_quantize_layer_workspace_size", "nvfp4_quantize_layer", "nvfp4_quantize_layer_order",
    "quantize_layer_many", "nvfp4_gptq_workspace_size", "nvfp4_gptq_quantize", "gptq_quantize",
    "nvfp4_scale_sweep_quantize_f32", "scale_sweep_quantize_f32", "nvfp4_gptq_set_timing",
    "nvfp4_gptq_phase_times", "GPTQ_PHASES", "nvfp4_debug_checks", "nvfp4_debug_checks_compiled", "Layer", "nvfp4_quantize_layers_workspace_size",
    "nvfp4_quantize_layers", "quantize_layers_many", "quantize_grouped_layer",
    "LayerWeight", "LayerInput", "GroupedInput", "nvfp4_quantize_grouped_layer_workspace_size",
    "nvfp4_quantize_grouped_layer", "nvfp4_quantize_grouped_layer_order",
    "diag_hessian_grouped", "global_scale_batched", "scale_sweep_quantize_batched",
    "nvfp4_scale_sweep_quantize", "nvfp4_dequantize", "nvfp4_quantize_activations",
    "quantize_activations", "nvfp4_blocked_scales_size", "nvfp4_scales_to_blocked",
    "scales_to_blocked",
    "diag_hessian", "global_scale", "scale_sweep_quantize", "dequantize", "quantize_layer",
]

STATUS = {0: "NVFP4_OK", -1: "NVFP4_ERR_INVALID_ARG", -2: "NVFP4_ERR_SHAPE",
          -3: "NVFP4_ERR_ALIGN", -4: "NVFP4_ERR_WINDOW", -5: "NVFP4_ERR_NONFINITE",
          -6: "NVFP4_ERR_CUDA", -7: "NVFP4_ERR_WORKSPACE", -8: "NVFP4_ERR_CAPTURE",
          -9: "NVFP4_ERR_NUMERIC"}


class NVFP4Error(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        self.status = status
        msg = f"{fn} returned {status} ({STATUS.get(status, '?')})"
        if status == -6:
            msg += f", cudaError {cuda_error}"
        super().__init__(msg)


_lock = threading.Lock()
_lib = None
LIB_PATH = _build.LIB

_vp, _i64, _sz, _int, _f32 = C.c_void_p, C.c_int64, C.c_size_t, C.c_int, C.c_float


class MatrixDesc(C.Structure):
    """nvfp4_matrix_desc"""
    _fields_ = [("W", _vp), ("out", _i64), ("inp", _i64), ("ldw", _i64)]


class SweepDesc(C.Structure):
    """nvfp4_sweep_desc"""
    _fields_ = [("W", _vp), ("out", _i64), ("inp", _i64), ("ldw", _i64), ("h", _vp), ("S", _vp),
                ("codes", _vp), ("scales", _vp), ("chosen_offset", _vp)]


class LayerWeight(C.Structure):
    """nvfp4_layer_weight"""
    _fields_ = [("W", _vp), ("out", _i64), ("inp", _i64), ("ldw", _i64), ("input", _int),
                ("S", _vp), ("amax", _vp), ("status", _vp), ("codes", _vp), ("scales", _vp),
                ("chosen_offset", _vp)]


class LayerInput(C.Structure):
    """nvfp4_layer_input"""
    _fields_ = [("X", _vp), ("tokens", _i64), ("inp", _i64), ("ldx", _i64), ("h", _vp)]


class Layer(C.Structure):
    """nvfp4_layer: one layer's weight and input descriptors"""
    _fields_ = [("weights", C.POINTER(LayerWeight)), ("n_weights", _int),
                ("inputs", C.POINTER(LayerInput)), ("n_inputs", _int)]


class GroupedInput(C.Structure):
    """nvfp4_grouped_input"""
    _fields_ = [("X", _vp), ("row_offsets", _vp), ("total_tokens", _i64), ("inp", _i64),
                ("ldx", _i64), ("h", _vp)]


_SIGS = {
    "nvfp4_version": ([], _int),
    "nvfp4_last_cuda_error": ([], _int),
    "nvfp4_debug_checks_compiled": ([], _int),
    "nvfp4_debug_checks": ([C.POINTER(C.c_ulonglong), C.POINTER(C.c_uint), _int], _int),
    "nvfp4_diag_hessian_workspace_size": ([_i64, _i64], _sz),
    "nvfp4_diag_hessian": ([_vp, _i64, _i64, _i64, _vp, _int, _vp, _sz, _vp], _int),
    "nvfp4_global_scale_workspace_size": ([_i64, _i64], _sz),
    "nvfp4_global_scale": ([_vp, _i64, _i64, _i64, _f32, _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "nvfp4_global_scale_noalloc": ([_vp, _i64, _i64, _i64, _f32, _vp, _vp, _vp, _vp], _int),
    "nvfp4_scale_sweep_quantize": ([_vp, _i64, _i64, _i64, _vp, _vp, _int, _int, _vp, _vp, _vp,
                                    _vp], _int),
    "nvfp4_debug_row_counters": ([C.POINTER(_vp), C.POINTER(_sz)], _int),
    "nvfp4_quantize_grouped_layer_workspace_size": ([C.POINTER(SweepDesc), _i64, C.POINTER(SweepDesc),
                                                     _i64, C.POINTER(GroupedInput),
                                                     C.POINTER(GroupedInput), _i64, _vp], _sz),
    "nvfp4_quantize_grouped_layer_order": ([C.POINTER(SweepDesc), _i64, C.POINTER(SweepDesc), _i64,
                                            C.POINTER(GroupedInput), C.POINTER(GroupedInput), _i64,
                                            _vp, _int, _int], _int),
    "nvfp4_quantize_grouped_layer": ([C.POINTER(SweepDesc), _i64, C.POINTER(SweepDesc), _i64,
                                      C.POINTER(GroupedInput), C.POINTER(GroupedInput), _i64, _f32,
                                      _int, _int, _vp, _vp, _vp, _vp, _sz, C.POINTER(_vp), _vp],
                                     _int),
    "nvfp4_quantize_layer_workspace_size": ([C.POINTER(LayerWeight), _int, C.POINTER(LayerInput),
                                             _int], _sz),
    "nvfp4_quantize_layer_order": ([C.POINTER(LayerWeight), _int, C.POINTER(LayerInput), _int, _int,
                                    _int, C.POINTER(_int)], _int),
    "nvfp4_quantize_layer": ([C.POINTER(LayerWeight), _int, C.POINTER(LayerInput), _int, _f32, _int,
                              _int, _vp, _sz, C.POINTER(_vp), _vp], _int),
    "nvfp4_quantize_layers_workspace_size": ([C.POINTER(Layer), _int], _sz),
    "nvfp4_quantize_layers": ([C.POINTER(Layer), _int, _f32, _int, _int, _vp, _sz, C.POINTER(_vp),
                               _vp], _int),
    "nvfp4_dequantize": ([_vp, _vp, _vp, _i64, _i64, _vp, _vp], _int),
    "nvfp4_gptq_workspace_size": ([_i64, _i64, _i64], _sz),
    "nvfp4_gptq_quantize": ([_vp, _i64, _i64, _i64, _vp, _i64, _i64, _f32, _int, _int, _f32, _int,
                             _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "nvfp4_scale_sweep_quantize_f32": ([_vp, _i64, _i64, _i64, _vp, _vp, _int, _int, _vp, _vp, _vp],
                                       _int),
    "nvfp4_gptq_set_timing": ([_int], _int),
    "nvfp4_gptq_phase_times": ([C.POINTER(C.c_float), _int], _int),
    "nvfp4_blocked_scales_size": ([_i64, _i64], _sz),
    "nvfp4_scales_to_blocked": ([_vp, _i64, _i64, _i64, _vp, _vp], _int),
    "nvfp4_quantize_activations": ([_vp, _i64, _i64, _i64, _f32, _int, _int, _vp, _vp, _vp, _vp,
                                    _vp, _vp], _int),
    "nvfp4_scale_sweep_quantize_full": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp],
                                        _int),
    "nvfp4_diag_hessian_grouped_workspace_size": ([_i64, _i64, _i64], _sz),
    "nvfp4_diag_hessian_grouped": ([_vp, _vp, _i64, _i64, _i64, _i64, _vp, _int, _vp, _sz, _vp],
                                   _int),
    "nvfp4_global_scale_batched_workspace_size": ([C.POINTER(MatrixDesc), _i64], _sz),
    "nvfp4_global_scale_batched": ([C.POINTER(MatrixDesc), _i64, _f32, _vp, _vp, _vp, _vp, _sz,
                                    _vp], _int),
    "nvfp4_scale_sweep_quantize_batched_workspace_size": ([_i64], _sz),
    "nvfp4_scale_sweep_quantize_batched": ([C.POINTER(SweepDesc), _i64, _int, _int, _vp, _sz, _vp],
                                           _int),
}


def lib(path: str | None = None):
    """Load the shared library (built in-tree by ``__graft_entry__.build()``)."""
    global _lib
    with _lock:
        if _lib is None:
            # NVFP4HS_LIB selects another build of the library, e.g. the
            # bounds-checked libnvfp4hs_checked.so next to it
            p = path or os.environ.get("NVFP4HS_LIB") or LIB_PATH
            if not os.path.exists(p):
                raise ImportError(f"libnvfp4hs.so not built at {p}; run __graft_entry__.build()")
            L = C.CDLL(p)
            for name, (args, res) in _SIGS.items():
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = res
            _lib = L
    return _lib


def _check(fn: str, st: int):
    if st != 0:
        raise NVFP4Error(fn, st, lib().nvfp4_last_cuda_error() if st == -6 else 0)


def _ptr(t) -> int | None:
    if t is None or isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# ------------------------------------------------------------- raw C mirrors
# Same names and argument order as the C entry points; tensors (or None) stand
# in for pointers, and `stream` defaults to torch's current stream.

def nvfp4_version() -> int:
    return lib().nvfp4_version()


def nvfp4_diag_hessian_workspace_size(tokens: int, inp: int) -> int:
    return lib().nvfp4_diag_hessian_workspace_size(tokens, inp)


def nvfp4_diag_hessian(X, tokens, inp, ldx, h, accumulate, workspace, workspace_bytes, stream=None):
    _check("nvfp4_diag_hessian", lib().nvfp4_diag_hessian(
        _ptr(X), tokens, inp, ldx, _ptr(h), int(accumulate), _ptr(workspace), workspace_bytes,
        _stream(stream)))


def nvfp4_global_scale_workspace_size(out: int, inp: int) -> int:
    return lib().nvfp4_global_scale_workspace_size(out, inp)


def nvfp4_global_scale(W, out, inp, ldw, q_max, S, amax, status, workspace, workspace_bytes,
                       stream=None):
    _check("nvfp4_global_scale", lib().nvfp4_global_scale(
        _ptr(W), out, inp, ldw, float(q_max), _ptr(S), _ptr(amax), _ptr(status), _ptr(workspace),
        workspace_bytes, _stream(stream)))


def nvfp4_global_scale_noalloc(W, out, inp, ldw, q_max, S, amax, status, stream=None):
    """nvfp4_global_scale without a workspace, for callers that cannot
    allocate: the library's built-in 64 KiB device array holds the partial
    maxima.  Calls that overlap on the GPU share that array and race."""
    _check("nvfp4_global_scale_noalloc", lib().nvfp4_global_scale_noalloc(
        _ptr(W), out, inp, ldw, float(q_max), _ptr(S), _ptr(amax), _ptr(status), _stream(stream)))


def nvfp4_scale_sweep_quantize(W, out, inp, ldw, h, S, lo, hi, codes, scales, chosen_offset,
                               stream=None):
    _check("nvfp4_scale_sweep_quantize", lib().nvfp4_scale_sweep_quantize(
        _ptr(W), out, inp, ldw, _ptr(h), _ptr(S), int(lo), int(hi), _ptr(codes), _ptr(scales),
        _ptr(chosen_offset), _stream(stream)))


def _layer_arrays(weights, inputs):
    wa = (LayerWeight * max(1, len(weights)))(*weights)
    xa = (LayerInput * max(1, len(inputs)))(*inputs)
    return wa, xa


def nvfp4_quantize_layer_workspace_size(weights, inputs) -> int:
    """weights: list of LayerWeight, inputs: list of LayerInput."""
    wa, xa = _layer_arrays(weights, inputs)
    return lib().nvfp4_quantize_layer_workspace_size(wa, len(weights), xa, len(inputs))


def nvfp4_quantize_layer_order(weights, inputs, lo, hi) -> list[int]:
    """The order nvfp4_quantize_layer sweeps these weights in: element j is the
    index of the weight swept j-th (needs the device for its SM count)."""
    wa, xa = _layer_arrays(weights, inputs)
    order = (_int * max(1, len(weights)))()
    _check("nvfp4_quantize_layer_order", lib().nvfp4_quantize_layer_order(
        wa, len(weights), xa, len(inputs), int(lo), int(hi), order))
    return [int(order[j]) for j in range(len(weights))]


def nvfp4_quantize_layer(weights, inputs, q_max, lo, hi, workspace, workspace_bytes,
                         sweep_events=None, stream=None):
    """weights/inputs: lists of LayerWeight/LayerInput (or ready ctypes arrays);
    sweep_events: None or 2 * len(weights) torch.cuda.Event, recorded around
    each weight's sweep launch (torch creates a CUDA event at its first
    record, so record each once before passing it)."""
    if isinstance(weights, list):
        wa, xa = _layer_arrays(weights, inputs)
    else:
        wa, xa = weights, inputs
    ev = None
    if sweep_events is not None:
        ev = (_vp * len(sweep_events))(*[e.cuda_event for e in sweep_events])
    _check("nvfp4_quantize_layer", lib().nvfp4_quantize_layer(
        wa, len(weights), xa, len(inputs), float(q_max), int(lo), int(hi), _ptr(workspace),
        workspace_bytes, ev, _stream(stream)))


def _layers_array(layers):
    """layers: list of (weights, inputs) lists of LayerWeight / LayerInput.
    Returns the ctypes array and the per-layer arrays it points into (which
    must outlive the call)."""
    keep = [_layer_arrays(w, x) for w, x in layers]
    arr = (Layer * max(1, len(layers)))(*[Layer(wa, len(w), xa, len(x))
                                          for (wa, xa), (w, x) in zip(keep, layers)])
    return arr, keep


def nvfp4_quantize_layers_workspace_size(layers) -> int:
    arr, _keep = _layers_array(layers)
    return lib().nvfp4_quantize_layers_workspace_size(arr, len(layers))


def nvfp4_quantize_layers(layers, q_max, lo, hi, workspace, workspace_bytes, sweep_events=None,
                          stream=None):
    """layers: list of (weights, inputs), as for nvfp4_quantize_layer; a weight's
    input indexes its own layer's inputs."""
    arr, _keep = _layers_array(layers)
    ev = None
    if sweep_events is not None:
        ev = (_vp * len(sweep_events))(*[e.cuda_event for e in sweep_events])
    _check("nvfp4_quantize_layers", lib().nvfp4_quantize_layers(
        arr, len(layers), float(q_max), int(lo), int(hi), _ptr(workspace), workspace_bytes, ev,
        _stream(stream)))


def _sweep_array(descs):
    return descs if not isinstance(descs, list) else (SweepDesc * max(1, len(descs)))(*descs)


def nvfp4_quantize_grouped_layer_workspace_size(first, second, first_input, second_input,
                                                experts, S) -> int:
    fa, sa = _sweep_array(first), _sweep_array(second)
    return lib().nvfp4_quantize_grouped_layer_workspace_size(
        fa, len(first), sa, len(second), C.byref(first_input), C.byref(second_input), experts,
        _ptr(S))


def nvfp4_quantize_grouped_layer_order(first, second, first_input, second_input, experts, S,
                                       lo, hi) -> int:
    """0 if nvfp4_quantize_grouped_layer with these arguments sweeps `first`
    first, 1 if it sweeps `second` first (host only, no CUDA call)."""
    fa, sa = _sweep_array(first), _sweep_array(second)
    r = lib().nvfp4_quantize_grouped_layer_order(
        fa, len(first), sa, len(second), C.byref(first_input), C.byref(second_input), experts,
        _ptr(S), int(lo), int(hi))
    _check("nvfp4_quantize_grouped_layer_order", min(r, 0))
    return r


def nvfp4_quantize_grouped_layer(first, second, first_input, second_input, experts, q_max, lo, hi,
                                 S, amax, status, workspace, workspace_bytes, sweep_events=None,
                                 stream=None):
    """first/second: lists (or ready ctypes arrays) of SweepDesc; first_input,
    second_input: GroupedInput; sweep_events: None or 4 recorded-once
    torch.cuda.Event around the two batches' sweep launches."""
    fa, sa = _sweep_array(first), _sweep_array(second)
    ev = None
    if sweep_events is not None:
        ev = (_vp * 4)(*[e.cuda_event for e in sweep_events])
    _check("nvfp4_quantize_grouped_layer", lib().nvfp4_quantize_grouped_layer(
        fa, len(first), sa, len(second), C.byref(first_input), C.byref(second_input), experts,
        float(q_max), int(lo), int(hi), _ptr(S), _ptr(amax), _ptr(status), _ptr(workspace),
        workspace_bytes, ev, _stream(stream)))


def nvfp4_gptq_workspace_size(out: int, inp: int, tokens: int) -> int:
    return lib().nvfp4_gptq_workspace_size(out, inp, tokens)


def nvfp4_gptq_quantize(W, out, inp, ldw, X, tokens, ldx, q_max, lo, hi, damp, weighted, codes,
                        scales, S, h, status, workspace, workspace_bytes, stream=None):
    _check("nvfp4_gptq_quantize", lib().nvfp4_gptq_quantize(
        _ptr(W), out, inp, ldw, _ptr(X), tokens, ldx, float(q_max), int(lo), int(hi), float(damp),
        int(bool(weighted)), _ptr(codes), _ptr(scales), _ptr(S), _ptr(h), _ptr(status),
        _ptr(workspace), workspace_bytes, _stream(stream)))


GPTQ_PHASES = ("reductions", "gram", "factor", "batch", "split", "update")


def nvfp4_gptq_set_timing(on: bool) -> None:
    _check("nvfp4_gptq_set_timing", lib().nvfp4_gptq_set_timing(int(bool(on))))


def nvfp4_gptq_phase_times() -> dict:
    """Milliseconds per GPTQ phase summed over the calls timed since
    nvfp4_gptq_set_timing(True) (waits for their events)."""
    ms = (C.c_float * len(GPTQ_PHASES))()
    _check("nvfp4_gptq_phase_times", lib().nvfp4_gptq_phase_times(ms, len(GPTQ_PHASES)))
    return {name: float(ms[i]) for i, name in enumerate(GPTQ_PHASES)}


def nvfp4_scale_sweep_quantize_f32(W, out, inp, ldw, h, S, lo, hi, codes, scales, stream=None):
    _check("nvfp4_scale_sweep_quantize_f32", lib().nvfp4_scale_sweep_quantize_f32(
        _ptr(W), out, inp, ldw, _ptr(h), _ptr(S), int(lo), int(hi), _ptr(codes), _ptr(scales),
        _stream(stream)))


def nvfp4_debug_checks_compiled() -> bool:
    """Whether this build of the library checks its global accesses."""
    return bool(lib().nvfp4_debug_checks_compiled())


def nvfp4_debug_checks(reset: bool = False):
    """(failed checks, first failure) of a bounds-checked build; (0, 0) for a
    build without checks (see nvfp4_debug_checks_compiled)."""
    first, count = C.c_ulonglong(0), C.c_uint(0)
    _check("nvfp4_debug_checks", lib().nvfp4_debug_checks(C.byref(first), C.byref(count),
                                                          int(bool(reset))))
    return count.value, first.value


def nvfp4_debug_row_counters():
    """(device address, bytes) of the sweep's run-time row counters on the
    current device; for tests only."""
    p, n = _vp(), _sz()
    _check("nvfp4_debug_row_counters", lib().nvfp4_debug_row_counters(C.byref(p), C.byref(n)))
    return p.value, n.value


def nvfp4_scale_sweep_quantize_full(W, out, inp, ldw, h, S, codes, scales, chosen_offset,
                                    stream=None):
    _check("nvfp4_scale_sweep_quantize_full", lib().nvfp4_scale_sweep_quantize_full(
        _ptr(W), out, inp, ldw, _ptr(h), _ptr(S), _ptr(codes), _ptr(scales), _ptr(chosen_offset),
        _stream(stream)))


def nvfp4_quantize_activations(A, tokens, inp, lda, q_max, lo, hi, S, codes, scales,
                               chosen_offset, status, stream=None):
    _check("nvfp4_quantize_activations", lib().nvfp4_quantize_activations(
        _ptr(A), tokens, inp, lda, float(q_max), int(lo), int(hi), _ptr(S), _ptr(codes),
        _ptr(scales), _ptr(chosen_offset), _ptr(status), _stream(stream)))


def nvfp4_blocked_scales_size(rows: int, cols: int) -> int:
    return lib().nvfp4_blocked_scales_size(rows, cols)


def nvfp4_scales_to_blocked(scales, rows, cols, ld, out, stream=None):
    _check("nvfp4_scales_to_blocked", lib().nvfp4_scales_to_blocked(
        _ptr(scales), rows, cols, ld, _ptr(out), _stream(stream)))


def nvfp4_dequantize(codes, scales, S, out, inp, W_out, stream=None):
    _check("nvfp4_dequantize", lib().nvfp4_dequantize(
        _ptr(codes), _ptr(scales), _ptr(S), out, inp, _ptr(W_out), _stream(stream)))


def nvfp4_diag_hessian_grouped_workspace_size(total_tokens: int, experts: int, inp: int) -> int:
    return lib().nvfp4_diag_hessian_grouped_workspace_size(total_tokens, experts, inp)


def nvfp4_diag_hessian_grouped(X, row_offsets, experts, total_tokens, inp, ldx, h, accumulate,
                               workspace, workspace_bytes, stream=None):
    _check("nvfp4_diag_hessian_grouped", lib().nvfp4_diag_hessian_grouped(
        _ptr(X), _ptr(row_offsets), experts, total_tokens, inp, ldx, _ptr(h), int(accumulate),
        _ptr(workspace), workspace_bytes, _stream(stream)))


def _desc_array(cls, items):
    arr = (cls * max(1, len(items)))()
    for i, it in enumerate(items):
        arr[i] = it
    return arr


def nvfp4_global_scale_batched_workspace_size(descs) -> int:
    arr = _desc_array(MatrixDesc, descs)
    return lib().nvfp4_global_scale_batched_workspace_size(arr, len(descs))


def nvfp4_global_scale_batched(descs, q_max, S, amax, status, workspace, workspace_bytes,
                               stream=None):
    arr = _desc_array(MatrixDesc, descs)
    _check("nvfp4_global_scale_batched", lib().nvfp4_global_scale_batched(
        arr, len(descs), float(q_max), _ptr(S), _ptr(amax), _ptr(status), _ptr(workspace),
        workspace_bytes, _stream(stream)))


def nvfp4_scale_sweep_quantize_batched_workspace_size(n: int) -> int:
    return lib().nvfp4_scale_sweep_quantize_batched_workspace_size(n)


def nvfp4_scale_sweep_quantize_batched(descs, lo, hi, workspace, workspace_bytes, stream=None):
    arr = _desc_array(SweepDesc, descs)
    _check("nvfp4_scale_sweep_quantize_batched", lib().nvfp4_scale_sweep_quantize_batched(
        arr, len(descs), int(lo), int(hi), _ptr(workspace), workspace_bytes, _stream(stream)))


# -------------------------------------------------------- tensor conveniences

def _bf16_2d(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or t.dim() != 2 or not t.is_cuda:
        raise ValueError(f"{name} must be a 2-D bf16 CUDA tensor")
    if t.stride(1) != 1:
        raise ValueError(f"{name} must have unit stride along its last dimension")
    return t


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def diag_hessian(X: torch.Tensor, h: torch.Tensor | None = None, accumulate: bool = False,
                 workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """h[in] (+)= sum_t X[t, :]^2 (float32)."""
    X = _bf16_2d(X, "X")
    T, n = X.shape
    if h is None:
        h = torch.empty(n, dtype=torch.float32, device=X.device)
    nb = nvfp4_diag_hessian_workspace_size(T, n)
    if nb == 0:
        raise NVFP4Error("nvfp4_diag_hessian_workspace_size", -1)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, X.device)
    nvfp4_diag_hessian(X, T, n, X.stride(0), h, accumulate, ws, ws.numel(), stream)
    return h


def global_scale(W: torch.Tensor, q_max: float = 448.0, workspace: torch.Tensor | None = None,
                 stream=None):
    """Returns device tensors (S[1], amax[1], status[1] int32)."""
    W = _bf16_2d(W, "W")
    o, n = W.shape
    dev = W.device
    S = torch.empty(1, dtype=torch.float32, device=dev)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    status = torch.empty(1, dtype=torch.int32, device=dev)
    nb = nvfp4_global_scale_workspace_size(o, n)
    if nb == 0:
        raise NVFP4Error("nvfp4_global_scale_workspace_size", -1)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, dev)
    nvfp4_global_scale(W, o, n, W.stride(0), q_max, S, amax, status, ws, ws.numel(), stream)
    return S, amax, status


def scale_sweep_quantize(W: torch.Tensor, h: torch.Tensor | None, S: torch.Tensor, lo: int = -9,
                         hi: int = 6, want_offsets: bool = False, out=None, stream=None):
    """Returns (codes[out, in/2] u8, scales[out, in/16] u8, offsets or None)."""
    W = _bf16_2d(W, "W")
    o, n = W.shape
    dev = W.device
    if out is None:
        codes = torch.empty(o, n // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(o, n // 16, dtype=torch.uint8, device=dev)
        offs = torch.empty(o, n // 16, dtype=torch.int8, device=dev) if want_offsets else None
    else:
        codes, scales, offs = out
    nvfp4_scale_sweep_quantize(W, o, n, W.stride(0), h, S, lo, hi, codes, scales, offs, stream)
    return codes, scales, offs


def scale_sweep_quantize_full(W: torch.Tensor, h: torch.Tensor | None, S: torch.Tensor,
                              want_offsets: bool = False, stream=None):
    """Sweep over all 126 positive E4M3 codes: (codes, scales, offsets or None)."""
    W = _bf16_2d(W, "W")
    o, n = W.shape
    codes = torch.empty(o, n // 2, dtype=torch.uint8, device=W.device)
    scales = torch.empty(o, n // 16, dtype=torch.uint8, device=W.device)
    offs = torch.empty(o, n // 16, dtype=torch.int8, device=W.device) if want_offsets else None
    nvfp4_scale_sweep_quantize_full(W, o, n, W.stride(0), h, S, codes, scales, offs, stream)
    return codes, scales, offs


def dequantize(codes: torch.Tensor, scales: torch.Tensor, S: torch.Tensor, stream=None):
    o, half = codes.shape
    W = torch.empty(o, half * 2, dtype=torch.float32, device=codes.device)
    nvfp4_dequantize(codes, scales, S, o, half * 2, W, stream)
    return W


def quantize_activations(A: torch.Tensor, q_max: float = 256.0, lo: int = -3, hi: int = 7,
                         want_offsets: bool = False, out=None, stream=None):
    """Per-token NVFP4 quantization of activations A[tokens, in] in one launch.
    Returns (S[tokens] f32, codes[tokens, in/2] u8, scales[tokens, in/16] u8,
    offsets or None, status[1] int32)."""
    A = _bf16_2d(A, "A")
    t, n = A.shape
    dev = A.device
    if out is None:
        S = torch.empty(t, dtype=torch.float32, device=dev)
        codes = torch.empty(t, n // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(t, n // 16, dtype=torch.uint8, device=dev)
        offs = torch.empty(t, n // 16, dtype=torch.int8, device=dev) if want_offsets else None
        status = torch.empty(1, dtype=torch.int32, device=dev)
    else:
        S, codes, scales, offs, status = out
    nvfp4_quantize_activations(A, t, n, A.stride(0), q_max, lo, hi, S, codes, scales, offs, status,
                               stream)
    return S, codes, scales, offs, status


def scales_to_blocked(scales: torch.Tensor, stream=None) -> torch.Tensor:
    """Row-major scale bytes [rows, in/16] -> the tensor-core tiled layout
    (flat uint8, rows padded to 128 and columns to 4)."""
    rows, cols = scales.shape
    out = torch.empty(max(16, nvfp4_blocked_scales_size(rows, cols)), dtype=torch.uint8,
                      device=scales.device)
    nvfp4_scales_to_blocked(scales, rows, cols, scales.stride(0), out, stream)
    return out[:nvfp4_blocked_scales_size(rows, cols)]


def quantize_layer(W: torch.Tensor, X: torch.Tensor | None, q_max: float = 448.0, lo: int = -9,
                   hi: int = 6, stream=None):
    """The whole path for one layer: h from X (None = plain MSE), S from W,
    then the windowed sweep.  Returns (codes, scales, S, h)."""
    h = diag_hessian(X, stream=stream) if X is not None else None
    S, _, _ = global_scale(W, q_max, stream=stream)
    codes, scales, _ = scale_sweep_quantize(W, h, S, lo, hi, stream=stream)
    return codes, scales, S, h


def quantize_layer_many(Ws, Xs, inputs, q_max: float = 448.0, lo: int = -9, hi: int = 6,
                        want_offsets: bool = False, stream=None):
    """Several projections of one layer in one call (nvfp4_quantize_layer).
    Ws: bf16 weights; Xs: bf16 calibration inputs; inputs[j]: index into Xs of
    W_j's input, or -1 for plain MSE.  Returns (list of (codes, scales, S,
    offsets or None, status) per weight, list of h per input)."""
    Ws = [_bf16_2d(W, "W") for W in Ws]
    Xs = [_bf16_2d(X, "X") for X in Xs]
    dev = (Ws or Xs)[0].device
    hs = [torch.empty(X.shape[1], dtype=torch.float32, device=dev) for X in Xs]
    outs, wd = [], []
    for W, k in zip(Ws, inputs):
        o, n = W.shape
        codes = torch.empty(o, n // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(o, n // 16, dtype=torch.uint8, device=dev)
        S = torch.empty(1, dtype=torch.float32, device=dev)
        status = torch.empty(1, dtype=torch.int32, device=dev)
        offs = torch.empty(o, n // 16, dtype=torch.int8, device=dev) if want_offsets else None
        wd.append(LayerWeight(W.data_ptr(), o, n, W.stride(0), int(k), S.data_ptr(), None,
                              status.data_ptr(), codes.data_ptr(), scales.data_ptr(), _ptr(offs)))
        outs.append((codes, scales, S, offs, status))
    xd = [LayerInput(X.data_ptr(), X.shape[0], X.shape[1], X.stride(0), h.data_ptr())
          for X, h in zip(Xs, hs)]
    nb = nvfp4_quantize_layer_workspace_size(wd, xd)
    if nb == 0:
        raise NVFP4Error("nvfp4_quantize_layer_workspace_size", -1)
    ws = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
    base = (-ws.data_ptr()) % 256
    wsv = ws[base:base + nb]
    nvfp4_quantize_layer(wd, xd, q_max, lo, hi, wsv, nb, stream)
    return outs, hs


def quantize_grouped_layer(first, second, first_input, second_input, row_offsets,
                           q_max: float = 448.0, lo: int = -9, hi: int = 6, weighted: bool = True,
                           want_offsets: bool = False, stream=None):
    """A mixture-of-experts layer in one call (nvfp4_quantize_grouped_layer).
    first, second: lists of (W, expert) -- bf16 weights and the expert whose
    row of the first (resp. second) input's h weights them; first_input,
    second_input: expert-contiguous bf16 inputs; row_offsets: int64 CUDA
    tensor [E+1].  weighted=False sweeps both batches with plain MSE.
    Returns (outputs of first, outputs of second, h1 [E, in1], h2 [E, in2],
    S, amax, status), each output (codes, scales, offsets or None), S etc.
    device [n_first + n_second]."""
    X1 = _bf16_2d(first_input, "X")
    X2 = _bf16_2d(second_input, "X")
    dev = X1.device
    E = row_offsets.numel() - 1
    h1 = torch.empty(E, X1.shape[1], dtype=torch.float32, device=dev)
    h2 = torch.empty(E, X2.shape[1], dtype=torch.float32, device=dev)
    n = len(first) + len(second)
    S = torch.empty(n, dtype=torch.float32, device=dev)
    amax = torch.empty(n, dtype=torch.float32, device=dev)
    status = torch.empty(n, dtype=torch.int32, device=dev)
    descs, outs = ([], []), ([], [])
    for b, (batch, hb) in enumerate(((first, h1), (second, h2))):
        for W, e in batch:
            W = _bf16_2d(W, "W")
            o, k = W.shape
            i = len(descs[0]) if b == 0 else len(first) + len(descs[1])
            codes = torch.empty(o, k // 2, dtype=torch.uint8, device=dev)
            scales = torch.empty(o, k // 16, dtype=torch.uint8, device=dev)
            offs = torch.empty(o, k // 16, dtype=torch.int8, device=dev) if want_offsets else None
            descs[b].append(SweepDesc(W.data_ptr(), o, k, W.stride(0),
                                      hb[e].data_ptr() if weighted else None,
                                      S[i:i + 1].data_ptr(), codes.data_ptr(), scales.data_ptr(),
                                      _ptr(offs)))
            outs[b].append((codes, scales, offs))
    x1 = GroupedInput(X1.data_ptr(), row_offsets.data_ptr(), X1.shape[0], X1.shape[1],
                      X1.stride(0), h1.data_ptr())
    x2 = GroupedInput(X2.data_ptr(), row_offsets.data_ptr(), X2.shape[0], X2.shape[1],
                      X2.stride(0), h2.data_ptr())
    nb = nvfp4_quantize_grouped_layer_workspace_size(descs[0], descs[1], x1, x2, E, S)
    if nb == 0:
        raise NVFP4Error("nvfp4_quantize_grouped_layer_workspace_size", -1)
    ws = _workspace(nb, dev)
    nvfp4_quantize_grouped_layer(descs[0], descs[1], x1, x2, E, q_max, lo, hi, S, amax, status,
                                 ws, nb, stream=stream)
    return outs[0], outs[1], h1, h2, S, amax, status


def gptq_quantize(W: torch.Tensor, X: torch.Tensor, q_max: float = 448.0, lo: int = -9, hi: int = 6,
                  damp: float = 0.01, weighted: bool = True, stream=None):
    """GPTQ with the H-Scale local call (nvfp4_gptq_quantize).  Returns (codes,
    scales, S, h, status)."""
    W = _bf16_2d(W, "W")
    X = _bf16_2d(X, "X")
    o, n = W.shape
    dev = W.device
    codes = torch.empty(o, n // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(o, n // 16, dtype=torch.uint8, device=dev)
    S = torch.empty(1, dtype=torch.float32, device=dev)
    h = torch.empty(n, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    nb = nvfp4_gptq_workspace_size(o, n, X.shape[0])
    if nb == 0:
        raise NVFP4Error("nvfp4_gptq_workspace_size", -1)
    ws = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
    base = (-ws.data_ptr()) % 256
    nvfp4_gptq_quantize(W, o, n, W.stride(0), X, X.shape[0], X.stride(0), q_max, lo, hi, damp,
                        weighted, codes, scales, S, h, status, ws[base:base + nb], nb, stream)
    return codes, scales, S, h, status


def scale_sweep_quantize_f32(W: torch.Tensor, h: torch.Tensor | None, S: torch.Tensor,
                             lo: int = -9, hi: int = 6, stream=None):
    """The windowed sweep of an FP32 matrix (GPTQ's local call on its own)."""
    if W.dtype != torch.float32 or W.dim() != 2 or W.stride(1) != 1:
        raise ValueError("W must be a 2-D float32 CUDA tensor with unit inner stride")
    o, n = W.shape
    codes = torch.empty(o, n // 2, dtype=torch.uint8, device=W.device)
    scales = torch.empty(o, n // 16, dtype=torch.uint8, device=W.device)
    nvfp4_scale_sweep_quantize_f32(W, o, n, W.stride(0), h, S, lo, hi, codes, scales, stream)
    return codes, scales


def quantize_layers_many(layers, q_max: float = 448.0, lo: int = -9, hi: int = 6,
                         want_offsets: bool = False, stream=None):
    """Several consecutive layers in one call (nvfp4_quantize_layers).  layers:
    list of (Ws, Xs, inputs) as for quantize_layer_many.  Returns, per layer,
    (list of (codes, scales, S, offsets or None, status) per weight, list of h
    per input)."""
    descs, outs = [], []
    for Ws, Xs, inputs in layers:
        Ws = [_bf16_2d(W, "W") for W in Ws]
        Xs = [_bf16_2d(X, "X") for X in Xs]
        dev = (Ws or Xs)[0].device
        hs = [torch.empty(X.shape[1], dtype=torch.float32, device=dev) for X in Xs]
        lo_, wd = [], []
        for W, k in zip(Ws, inputs):
            o, n = W.shape
            codes = torch.empty(o, n // 2, dtype=torch.uint8, device=dev)
            scales = torch.empty(o, n // 16, dtype=torch.uint8, device=dev)
            S = torch.empty(1, dtype=torch.float32, device=dev)
            status = torch.empty(1, dtype=torch.int32, device=dev)
            offs = torch.empty(o, n // 16, dtype=torch.int8, device=dev) if want_offsets else None
            wd.append(LayerWeight(W.data_ptr(), o, n, W.stride(0), int(k), S.data_ptr(), None,
                                  status.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                                  _ptr(offs)))
            lo_.append((codes, scales, S, offs, status))
        xd = [LayerInput(X.data_ptr(), X.shape[0], X.shape[1], X.stride(0), h.data_ptr())
              for X, h in zip(Xs, hs)]
        descs.append((wd, xd))
        outs.append((lo_, hs))
    nb = nvfp4_quantize_layers_workspace_size(descs)
    if nb == 0:
        raise NVFP4Error("nvfp4_quantize_layers_workspace_size", -1)
    dev = outs[0][0][0][0].device if outs and outs[0][0] else outs[0][1][0].device
    ws = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
    base = (-ws.data_ptr()) % 256
    nvfp4_quantize_layers(descs, q_max, lo, hi, ws[base:base + nb], nb, stream=stream)
    return outs


def diag_hessian_grouped(X: torch.Tensor, row_offsets: torch.Tensor, h: torch.Tensor | None = None,
                         accumulate: bool = False, stream=None) -> torch.Tensor:
    """h[E, in]: per-expert sums of squares over expert-contiguous rows of X.
    row_offsets: int64 CUDA tensor [E+1]."""
    X = _bf16_2d(X, "X")
    T, n = X.shape
    E = row_offsets.numel() - 1
    if h is None:
        h = torch.empty(E, n, dtype=torch.float32, device=X.device)
    nb = nvfp4_diag_hessian_grouped_workspace_size(T, E, n)
    if nb == 0:
        raise NVFP4Error("nvfp4_diag_hessian_grouped_workspace_size", -1)
    ws = _workspace(nb, X.device)
    nvfp4_diag_hessian_grouped(X, row_offsets, E, T, n, X.stride(0), h, accumulate, ws, ws.numel(),
                               stream)
    return h


def global_scale_batched(Ws, q_max: float = 448.0, stream=None):
    """S, amax, status (device [n]) of many bf16 matrices in one launch."""
    descs = [MatrixDesc(_bf16_2d(W, "W").data_ptr(), W.shape[0], W.shape[1], W.stride(0)) for W in Ws]
    dev = Ws[0].device
    n = len(Ws)
    S = torch.empty(n, dtype=torch.float32, device=dev)
    amax = torch.empty(n, dtype=torch.float32, device=dev)
    status = torch.empty(n, dtype=torch.int32, device=dev)
    nb = nvfp4_global_scale_batched_workspace_size(descs)
    if nb == 0:
        raise NVFP4Error("nvfp4_global_scale_batched_workspace_size", -1)
    ws = _workspace(nb, dev)
    nvfp4_global_scale_batched(descs, q_max, S, amax, status, ws, ws.numel(), stream)
    return S, amax, status


def scale_sweep_quantize_batched(Ws, hs, Ss, lo: int = -9, hi: int = 6, want_offsets=False,
                                 stream=None):
    """Sweep many matrices in one launch.  hs: list of h (or None for all),
    Ss: list of device scalars (e.g. views into global_scale_batched's S)."""
    descs, outs = [], []
    for i, W in enumerate(Ws):
        W = _bf16_2d(W, "W")
        o, n = W.shape
        codes = torch.empty(o, n // 2, dtype=torch.uint8, device=W.device)
        scales = torch.empty(o, n // 16, dtype=torch.uint8, device=W.device)
        offs = torch.empty(o, n // 16, dtype=torch.int8, device=W.device) if want_offsets else None
        h = None if hs is None else hs[i]
        descs.append(SweepDesc(W.data_ptr(), o, n, W.stride(0), _ptr(h), Ss[i].data_ptr(),
                               codes.data_ptr(), scales.data_ptr(), _ptr(offs)))
        outs.append((codes, scales, offs))
    nb = nvfp4_scale_sweep_quantize_batched_workspace_size(len(descs))
    ws = _workspace(nb, Ws[0].device)
    nvfp4_scale_sweep_quantize_batched(descs, lo, hi, ws, ws.numel(), stream)
    return outs
