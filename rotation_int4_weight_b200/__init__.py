"""Python binding of libparo, the C ABI of the ParoQuant runtime hot path on B200.

Argument marshalling only: every function forwards device pointers, sizes and
the current CUDA stream to the entry point of the same name in libparo.so
(declared in include/paro.h) and raises ParoError on a non-OK status.  Output
tensors are allocated here with torch when the caller passes none; no step of
the computation runs in Python.  Importing this module fails loudly when the
library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "ParoError", "LIB_PATH", "lib", "paro_weight_layout_version", "paro_workspace_bytes",
    "paro_pack_weights", "paro_rotate", "paro_w4_linear", "paro_rotate_w4_linear",
    "paro_rotate_w4_linear_noalloc", "paro_get_device_status", "EXPORTED", "ParoLinear", "paro_linear",
    "paro_batched_workspace_bytes", "paro_rotate_w4_linear_batched", "paro_plan_pair_order",
    "paro_rotate_backward_workspace_bytes", "paro_rotate_backward", "paro_set_test_hooks", "paro_dense_rotate",
    "paro_quantize_activations", "paro_w4a4_linear", "paro_rotate_w4a4_linear",
]

# PARO_TIMELINE=1 loads the instrumented build (same kernels plus global-timer
# stamps of the fused one-token decode launch; built by _build.py --timeline)
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libparo_timeline.so" if os.environ.get("PARO_TIMELINE") == "1" else "libparo.so")

# name -> (restype, argtypes) of every entry point of include/paro.h
_P, _I, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
EXPORTED = {
    "paro_weight_layout_version": (_I, []),
    "paro_status_string": (ctypes.c_char_p, [_I]),
    "paro_last_error": (ctypes.c_char_p, []),
    "paro_pack_weights": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "paro_rotate": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "paro_w4_linear": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "paro_workspace_bytes": (_S, [_I, _I]),
    "paro_rotate_w4_linear": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
    "paro_rotate_w4_linear_noalloc": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "paro_batched_workspace_bytes": (_S, [_P, _I]),
    "paro_rotate_w4_linear_batched": (_I, [_P, _I, _I, _P, _S, _P]),
    "paro_plan_pair_order": (_I, [_P, _P, _P, _I, _I, _P, _P, _P]),
    "paro_get_device_status": (_I, [_P]),
    "paro_rotate_backward_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "paro_rotate_backward": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "paro_set_test_hooks": (_I, [ctypes.c_longlong, _I]),
    "paro_dense_rotate": (_I, [_P, _P, _P, _I, _I, _P]),
    "paro_quantize_activations": (_I, [_P, _P, _P, _I, _I, _P]),
    "paro_w4a4_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "paro_w4a4_linear": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
    "paro_rotate_w4a4_linear": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
}


class ParoLinear(ctypes.Structure):
    """Host-side description of one linear (the C struct paro_linear)."""
    _fields_ = [("d_x", _P), ("d_y", _P), ("M", _I), ("d_in", _I), ("d_out", _I), ("K", _I),
                ("d_pairs", _P), ("d_cos", _P), ("d_sin", _P), ("d_scale", _P),
                ("d_qweight", _P), ("d_scales", _P), ("d_zeros", _P)]


class ParoError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(message)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python rotation_int4_weight_b200/_build.py` "
            "(there is no fallback implementation)")
    handle = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in EXPORTED.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    return handle


lib = _load()


def _check(status: int, what: str) -> None:
    if status != 0:
        name = lib.paro_status_string(status).decode()
        msg = lib.paro_last_error().decode()
        raise ParoError(status, f"{what}: {name}: {msg}")


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _u16(t: torch.Tensor) -> torch.Tensor:
    """bf16/fp16/int16/uint16 tensors all pass as 16-bit patterns."""
    if t.element_size() != 2:
        raise ValueError(f"expected a 16-bit tensor, got {t.dtype}")
    return t


def paro_weight_layout_version() -> int:
    return int(lib.paro_weight_layout_version())


def paro_workspace_bytes(M: int, d_in: int) -> int:
    return int(lib.paro_workspace_bytes(M, d_in))


def _K(pairs):
    return 0 if pairs is None else int(pairs.shape[0])


def paro_pack_weights(W: torch.Tensor, pairs=None, cos_t=None, sin_t=None, scale=None, *,
                      group_size: int = 128, workspace=None, qweight=None, scales=None, zeros=None,
                      stream=None):
    """Fold the layer's transform into fp32 W [d_out, d_in] and pack it (layout version 1).

    Returns (qweight int32 [d_out, d_in/8], scales fp16 [d_out, G], zeros fp16 [d_out, G]).
    """
    d_out, d_in = W.shape
    dev = W.device
    K = _K(pairs)
    if qweight is None:
        qweight = torch.empty(d_out, d_in // 8, dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty(d_out, max(d_in // 128, 1), dtype=torch.float16, device=dev)
    if zeros is None:
        zeros = torch.empty_like(scales)
    if workspace is None and (K > 0 or scale is not None):
        workspace = torch.empty(d_out, d_in, dtype=torch.float32, device=dev)
    st = lib.paro_pack_weights(_ptr(W), d_out, d_in, group_size, K, _ptr(pairs), _ptr(cos_t), _ptr(sin_t),
                               _ptr(scale), _ptr(workspace), _ptr(qweight), _ptr(_u16(scales)),
                               _ptr(_u16(zeros)), _stream(stream))
    _check(st, "paro_pack_weights")
    return qweight, scales, zeros


def paro_rotate(x: torch.Tensor, pairs=None, cos_t=None, sin_t=None, scale=None, *, out=None, stream=None):
    """x~ = diag(1/s) R_K ... R_1 x for bf16 x [M, d]; returns bf16 [M, d] (out may be x)."""
    M, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    st = lib.paro_rotate(_ptr(_u16(x)), _ptr(_u16(out)), M, d, _K(pairs), _ptr(pairs), _ptr(cos_t), _ptr(sin_t),
                         _ptr(scale), _stream(stream))
    _check(st, "paro_rotate")
    return out


def paro_rotate_backward(x: torch.Tensor, grad: torch.Tensor, pairs=None, cos_t=None, sin_t=None, scale=None, *,
                         workspace=None, stream=None):
    """Gradients of x~ = diag(1/s) R_K ... R_1 x for bf16 x [M, d] and fp32 grad = dL/dx~ [M, d].

    Returns (dx fp32 [M, d], dtheta fp32 [K, d/2] or None when K == 0, dscale fp32 [d] or None
    without a scale) and the workspace used (reusable).
    """
    M, d = x.shape
    K = _K(pairs)
    dx = torch.empty(M, d, dtype=torch.float32, device=x.device)
    dtheta = torch.empty(K, d // 2, dtype=torch.float32, device=x.device) if K else None
    dscale = torch.empty(d, dtype=torch.float32, device=x.device) if scale is not None else None
    need = lib.paro_rotate_backward_workspace_bytes(M, d, K, 1 if scale is not None else 0)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    st = lib.paro_rotate_backward(_ptr(_u16(x)), _ptr(grad), M, d, K, _ptr(pairs), _ptr(cos_t), _ptr(sin_t),
                                  _ptr(scale), _ptr(dx), _ptr(dtheta), _ptr(dscale), _ptr(workspace),
                                  workspace.numel(), _stream(stream))
    _check(st, "paro_rotate_backward")
    return (dx, dtheta, dscale), workspace


def paro_dense_rotate(x: torch.Tensor, q: torch.Tensor, *, out=None, stream=None):
    """The dense-rotation contrast: x~ = x Q^T for bf16 x [M, d] and bf16 Q [d, d]; bf16 [M, d]."""
    M, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    st = lib.paro_dense_rotate(_ptr(_u16(x)), _ptr(_u16(q)), _ptr(_u16(out)), M, d, _stream(stream))
    _check(st, "paro_dense_rotate")
    return out


def paro_quantize_activations(x: torch.Tensor, *, q=None, sx=None, stream=None):
    """Per-token symmetric INT4 codes of bf16 x [M, d]: (codes int8 [M, d] in -8..7, scales fp32 [M])."""
    M, d = x.shape
    if q is None:
        q = torch.empty(M, d, dtype=torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    st = lib.paro_quantize_activations(_ptr(_u16(x)), _ptr(q), _ptr(sx), M, d, _stream(stream))
    _check(st, "paro_quantize_activations")
    return q, sx


def _w4a4_ws(M, d_in, d_out, with_transform, workspace, dev):
    need = int(lib.paro_w4a4_workspace_bytes(M, d_in, d_out, with_transform))
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    return workspace, need


def paro_w4a4_linear(q: torch.Tensor, sx: torch.Tensor, qweight, scales, zeros, *, out=None, workspace=None,
                     group_size: int = 128, stream=None):
    """The W4A4 linear on activation codes q (int8 [M, d_in]) and scales sx (fp32 [M]); bf16 [M, d_out]."""
    M, d_in = q.shape
    d_out = qweight.shape[0]
    if out is None:
        out = torch.empty(M, d_out, dtype=torch.bfloat16, device=q.device)
    workspace, need = _w4a4_ws(M, d_in, d_out, 0, workspace, q.device)
    st = lib.paro_w4a4_linear(_ptr(q), _ptr(sx), _ptr(qweight), _ptr(_u16(scales)), _ptr(_u16(zeros)),
                              _ptr(_u16(out)), M, d_in, d_out, group_size, _ptr(workspace) if need else None,
                              workspace.numel() if need else 0, _stream(stream))
    _check(st, "paro_w4a4_linear")
    return out


def paro_rotate_w4a4_linear(x: torch.Tensor, pairs, cos_t, sin_t, scale, qweight, scales, zeros, *, out=None,
                            workspace=None, group_size: int = 128, stream=None):
    """The W4A4 path of one linear: transform, per-token INT4 codes, W4A4 linear; bf16 [M, d_out].
    The workspace (returned by paro_w4a4_workspace_bytes(M, d_in, d_out, 1)) holds x~ in bf16
    first, then its codes and scales."""
    M, d_in = x.shape
    d_out = qweight.shape[0]
    if out is None:
        out = torch.empty(M, d_out, dtype=torch.bfloat16, device=x.device)
    workspace, need = _w4a4_ws(M, d_in, d_out, 1, workspace, x.device)
    st = lib.paro_rotate_w4a4_linear(_ptr(_u16(x)), _K(pairs), _ptr(pairs), _ptr(cos_t), _ptr(sin_t), _ptr(scale),
                                     _ptr(qweight), _ptr(_u16(scales)), _ptr(_u16(zeros)), _ptr(_u16(out)), M, d_in,
                                     d_out, group_size, _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "paro_rotate_w4a4_linear")
    return out


def paro_w4_linear(x: torch.Tensor, qweight, scales, zeros, *, out=None, group_size: int = 128, stream=None):
    """y = x W^^T for bf16 x [M, d_in] and packed INT4 weights; returns bf16 [M, d_out]."""
    M, d_in = x.shape
    d_out = qweight.shape[0]
    if out is None:
        out = torch.empty(M, d_out, dtype=torch.bfloat16, device=x.device)
    st = lib.paro_w4_linear(_ptr(_u16(x)), _ptr(qweight), _ptr(_u16(scales)), _ptr(_u16(zeros)), _ptr(_u16(out)),
                            M, d_in, d_out, group_size, _stream(stream))
    _check(st, "paro_w4_linear")
    return out


def paro_rotate_w4_linear(x: torch.Tensor, pairs, cos_t, sin_t, scale, qweight, scales, zeros, *, out=None,
                          workspace=None, group_size: int = 128, stream=None):
    """The runtime path of one linear: transform x, then the packed INT4 linear; bf16 [M, d_out]."""
    M, d_in = x.shape
    d_out = qweight.shape[0]
    if out is None:
        out = torch.empty(M, d_out, dtype=torch.bfloat16, device=x.device)
    need = paro_workspace_bytes(M, d_in)
    if workspace is None:  # zero before its first use (the calls keep it valid afterwards)
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=x.device)
    st = lib.paro_rotate_w4_linear(_ptr(_u16(x)), _K(pairs), _ptr(pairs), _ptr(cos_t), _ptr(sin_t), _ptr(scale),
                                   _ptr(qweight), _ptr(_u16(scales)), _ptr(_u16(zeros)), _ptr(_u16(out)),
                                   M, d_in, d_out, group_size, _ptr(workspace), workspace.numel(),
                                   _stream(stream))
    _check(st, "paro_rotate_w4_linear")
    return out


def paro_rotate_w4_linear_noalloc(x: torch.Tensor, pairs, cos_t, sin_t, scale, qweight, scales, zeros, *,
                                  out=None, group_size: int = 128, stream=None):
    """paro_rotate_w4_linear without a workspace: the library's built-in scratch
    array holds the transformed activations, so the call allocates nothing
    (M * d_in <= 262144; calls that overlap on the GPU race on the array)."""
    M, d_in = x.shape
    d_out = qweight.shape[0]
    if out is None:
        out = torch.empty(M, d_out, dtype=torch.bfloat16, device=x.device)
    st = lib.paro_rotate_w4_linear_noalloc(_ptr(_u16(x)), _K(pairs), _ptr(pairs), _ptr(cos_t), _ptr(sin_t),
                                           _ptr(scale), _ptr(qweight), _ptr(_u16(scales)), _ptr(_u16(zeros)),
                                           _ptr(_u16(out)), M, d_in, d_out, group_size, _stream(stream))
    _check(st, "paro_rotate_w4_linear_noalloc")
    return out


def paro_linear(x, pairs, cos_t, sin_t, scale, qweight, scales, zeros, out) -> ParoLinear:
    """Describe one linear for paro_rotate_w4_linear_batched (tensors stay owned by the caller)."""
    def p(t):
        return None if t is None else _ptr(t).value
    return ParoLinear(p(_u16(x)), p(_u16(out)), x.shape[0], x.shape[1], qweight.shape[0], _K(pairs), p(pairs),
                      p(cos_t), p(sin_t), p(scale), p(qweight), p(_u16(scales)), p(_u16(zeros)))


def paro_batched_workspace_bytes(layers) -> int:
    arr = (ParoLinear * len(layers))(*layers)
    return int(lib.paro_batched_workspace_bytes(ctypes.cast(arr, ctypes.c_void_p), len(layers)))


def paro_rotate_w4_linear_batched(layers, *, workspace=None, group_size: int = 128, stream=None):
    """Run a list of ParoLinear descriptions (at most 8): one launch at one token
    per linear, a transform launch and an INT4-linear launch up to 64 tokens."""
    arr = (ParoLinear * len(layers))(*layers)
    need = int(lib.paro_batched_workspace_bytes(ctypes.cast(arr, ctypes.c_void_p), len(layers)))
    if workspace is None:  # zero before its first use (the calls keep it valid afterwards)
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")
    st = lib.paro_rotate_w4_linear_batched(ctypes.cast(arr, ctypes.c_void_p), len(layers), group_size,
                                           _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "paro_rotate_w4_linear_batched")
    return workspace


def paro_plan_pair_order(pairs, cos_t, sin_t):
    """Host-side: reorder (and flip) the pairs inside every stage for conflict-free
    shared-memory access; numpy arrays in ([K, d/2, 2] uint16, [K, d/2] fp32 x2),
    numpy arrays out describing the same transform."""
    import numpy as np
    pairs = np.ascontiguousarray(pairs, dtype=np.uint16)
    cos_t = np.ascontiguousarray(cos_t, dtype=np.float32)
    sin_t = np.ascontiguousarray(sin_t, dtype=np.float32)
    K, half = cos_t.shape
    po, co, so = np.empty_like(pairs), np.empty_like(cos_t), np.empty_like(sin_t)
    st = lib.paro_plan_pair_order(pairs.ctypes.data, cos_t.ctypes.data, sin_t.ctypes.data, K, 2 * half,
                                  po.ctypes.data, co.ctypes.data, so.ctypes.data)
    _check(st, "paro_plan_pair_order")
    return po, co, so


def paro_set_test_hooks(flag_wait_cycles: int = 0, skip_ready_flags: bool = False) -> None:
    """Test hooks of the failure paths: bound the decode INT4 kernel's hand-over
    flag waits to `flag_wait_cycles` SM cycles (0: the default, about a second)
    and make the decode transforms skip publishing their flags.  Affects the
    calls configured afterwards; (0, False) restores the defaults."""
    _check(lib.paro_set_test_hooks(int(flag_wait_cycles), 1 if skip_ready_flags else 0), "paro_set_test_hooks")


def paro_get_device_status(stream=None) -> int:
    """Synchronise the stream and return/clear the device status word (0 = OK)."""
    return int(lib.paro_get_device_status(_stream(stream)))
