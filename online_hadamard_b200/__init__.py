"""Python binding of libmacaq: the MACaQ MXFP4 W4A4 linear layer on B200 (sm_100a).

Argument marshalling only: every function below checks tensor placement, dtype and
contiguity, allocates outputs with torch when the caller does not pass them, and calls the
C entry point of the same name in ``_build/libmacaq.so`` with the tensors' device made
current, on that device's current CUDA stream (or the stream passed, which must belong to it).  All
arithmetic runs in the library's CUDA kernels; there is no CPU or PyTorch fallback -- if
the library cannot be loaded, every call raises.

Method: "MACaQ: Fast, Model Agnostic Calibrated Quantization for Low-Precision Weights and
Activations", Abstract (per-channel scale and block-Hadamard applied online to the
activations, inverse transforms absorbed into the weights, MXFP4 W4A4).  Layouts and
conventions are documented in include/macaq.h.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import torch

from . import build as _build_mod

__all__ = [
    "load_library", "MacaqError", "scale_bytes", "scale_offset", "linear_workspace_bytes", "gemm_workspace_bytes",
    "macaq_calibrate_scale", "macaq_fold_weights", "macaq_act_transform_quant", "macaq_act_quant_plain",
    "macaq_mxfp4_gemm", "macaq_w4a4_linear", "macaq_mxfp4_linear", "macaq_w4a4_grouped_linear",
    "grouped_workspace_bytes", "macaq_w4a4_linear_noalloc", "macaq_calib_hessian", "macaq_flip_refine",
    "macaq_w4a4_grouped_linear_device", "grouped_device_workspace_bytes", "macaq_scales_to_tiled",
    "macaq_scales_to_rowmajor", "macaq_w4a4_linear_multi", "linear_multi_workspace_bytes",
    "macaq_device_status", "status_str", "EXPORTED_SYMBOLS",
]

# Every symbol include/macaq.h declares.
EXPORTED_SYMBOLS = (
    "macaq_status_str", "macaq_scale_bytes", "macaq_scale_offset", "macaq_linear_workspace_bytes",
    "macaq_gemm_workspace_bytes",
    "macaq_calibrate_scale", "macaq_fold_weights", "macaq_act_transform_quant", "macaq_w4a4_linear",
    "macaq_act_quant_plain", "macaq_mxfp4_linear", "macaq_mxfp4_gemm", "macaq_device_status",
    "macaq_grouped_workspace_bytes", "macaq_w4a4_grouped_linear", "macaq_w4a4_linear_noalloc",
    "macaq_hessian_workspace_bytes", "macaq_calib_hessian", "macaq_flip_refine_workspace_bytes",
    "macaq_flip_refine", "macaq_grouped_device_workspace_bytes", "macaq_w4a4_grouped_linear_device",
    "macaq_scales_to_tiled", "macaq_scales_to_rowmajor", "macaq_linear_multi_workspace_bytes",
    "macaq_w4a4_linear_multi",
)

MACAQ_OK = 0

_lock = threading.Lock()
_lib = None


class MacaqError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_str(status)} ({status})")
        self.status = status


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if absent) libmacaq.so and declare its C signatures."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        lib_path = path or _build_mod.LIB_PATH
        if path is None and not os.path.exists(lib_path):
            _build_mod.build()
        lib = ctypes.CDLL(lib_path)
        p, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        lib.macaq_status_str.argtypes = [i32]
        lib.macaq_status_str.restype = ctypes.c_char_p
        lib.macaq_scale_bytes.argtypes = [i64, i64]
        lib.macaq_scale_bytes.restype = sz
        lib.macaq_scale_offset.argtypes = [i64, i64, i64]
        lib.macaq_scale_offset.restype = i64
        lib.macaq_linear_workspace_bytes.argtypes = [i64, i64, i64]
        lib.macaq_linear_workspace_bytes.restype = sz
        lib.macaq_gemm_workspace_bytes.argtypes = [i64, i64, i64]
        lib.macaq_gemm_workspace_bytes.restype = sz
        lib.macaq_calibrate_scale.argtypes = [p, i64, p, i64, i64, p, p]
        lib.macaq_fold_weights.argtypes = [p, i64, i64, p, p, p, p, p]
        lib.macaq_act_transform_quant.argtypes = [p, i64, i64, p, p, p, p]
        lib.macaq_act_quant_plain.argtypes = [p, i64, i64, p, p, p]
        lib.macaq_mxfp4_gemm.argtypes = [p, p, i64, p, p, i64, i64, p, i32, p, sz, p]
        lib.macaq_w4a4_linear.argtypes = [p, i64, i64, p, p, p, i64, p, p, sz, p]
        lib.macaq_mxfp4_linear.argtypes = [p, i64, i64, p, p, i64, p, p, sz, p]
        lib.macaq_grouped_workspace_bytes.argtypes = [p, i32, i64, i64]
        lib.macaq_grouped_workspace_bytes.restype = sz
        lib.macaq_w4a4_grouped_linear.argtypes = [p, p, i32, i64, p, p, p, i64, p, p, sz, p]
        lib.macaq_device_status.argtypes = [i32]
        lib.macaq_w4a4_linear_noalloc.argtypes = [p, i64, i64, p, p, p, i64, p, p]
        lib.macaq_hessian_workspace_bytes.argtypes = [i64, i64]
        lib.macaq_hessian_workspace_bytes.restype = sz
        lib.macaq_calib_hessian.argtypes = [p, i64, i64, p, p, p, sz, p]
        lib.macaq_flip_refine_workspace_bytes.argtypes = [i64, i64]
        lib.macaq_flip_refine_workspace_bytes.restype = sz
        lib.macaq_flip_refine.argtypes = [p, i64, i64, p, p, p, p, i64, p, p, sz, p]
        lib.macaq_scales_to_tiled.argtypes = [p, i64, i64, p, p]
        lib.macaq_scales_to_rowmajor.argtypes = [p, i64, i64, p, p]
        lib.macaq_grouped_device_workspace_bytes.argtypes = [i64, i32, i64, i64]
        lib.macaq_grouped_device_workspace_bytes.restype = sz
        lib.macaq_w4a4_grouped_linear_device.argtypes = [p, i64, p, i32, i32, i64, i64, p, p, p, i64, p, p, sz, p]
        lib.macaq_linear_multi_workspace_bytes.argtypes = [i64, i32, i64]
        lib.macaq_linear_multi_workspace_bytes.restype = sz
        lib.macaq_w4a4_linear_multi.argtypes = [p, i64, i64, i32, p, p, p, p, p, p, sz, p]
        for name in ("macaq_calibrate_scale", "macaq_fold_weights", "macaq_act_transform_quant", "macaq_act_quant_plain",
                     "macaq_mxfp4_gemm", "macaq_w4a4_linear", "macaq_mxfp4_linear", "macaq_device_status",
                     "macaq_w4a4_grouped_linear", "macaq_w4a4_linear_noalloc", "macaq_calib_hessian",
                     "macaq_flip_refine", "macaq_w4a4_grouped_linear_device", "macaq_scales_to_tiled",
                     "macaq_scales_to_rowmajor", "macaq_w4a4_linear_multi"):
            getattr(lib, name).restype = i32
        if path is None:
            _lib = lib
        return lib


def status_str(status: int) -> str:
    return load_library().macaq_status_str(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MACAQ_OK:
        raise MacaqError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device: torch.device) -> ctypes.c_void_p:
    """The CUDA stream handle of a call whose tensors live on `device`: the given stream, which
    must belong to that device, or that device's current stream."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    else:
        _check_stream_device(stream, device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check_stream_device(stream, device: torch.device) -> None:
    """A stream of another GPU would run the kernels there, on pointers into this one."""
    sdev = torch.device(stream.device)
    if sdev.type != "cuda" or sdev.index != device.index:
        raise ValueError(f"stream belongs to {sdev}, the call's tensors to {device}")


def _device(device):
    """`device` made current for the library call inside (None: the current device as it is)."""
    return contextlib.nullcontext() if device is None else torch.cuda.device(device)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None, min_numel=None, device=None) -> None:
    """Argument checks the C ABI cannot make (it sees bare pointers): a contiguous CUDA tensor of
    the right dtype and shape or size, on the device of the call's other tensors.  A buffer
    that is too small or on the wrong device would otherwise reach a kernel."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call's other tensors on {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_numel is not None:
        _need_numel(t, name, min_numel)


def _need_numel(t: torch.Tensor, name: str, n: int) -> None:
    if t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} elements, the call needs at least {n}")


def scale_bytes(rows: int, K: int) -> int:
    """Size of an E8M0 scale buffer in the MMA tile layout (include/macaq.h)."""
    return int(load_library().macaq_scale_bytes(rows, K))


def scale_offset(r: int, kb: int, K: int) -> int:
    return int(load_library().macaq_scale_offset(r, kb, K))


def linear_workspace_bytes(M: int, N: int, K: int, device=None) -> int:
    """Scratch bytes macaq_w4a4_linear and macaq_mxfp4_linear need on `device` (default: the
    current CUDA device; the size depends on its SM count)."""
    with _device(device):
        return int(load_library().macaq_linear_workspace_bytes(M, N, K))


def gemm_workspace_bytes(M: int, N: int, K: int, device=None) -> int:
    """Scratch bytes of the GEMM's stream-K schedule on `device` (default: the current one)."""
    with _device(device):
        return int(load_library().macaq_gemm_workspace_bytes(M, N, K))


def macaq_scales_to_tiled(rowmajor: torch.Tensor, K: int, tiled=None, stream=None):
    """Row-major E8M0 scales uint8 [rows, K/32] -> the MMA tile layout (uint8 [scale_bytes(rows, K)])."""
    rows = rowmajor.shape[0]
    _need(rowmajor, "rowmajor", torch.uint8, (rows, K // 32))
    dev = rowmajor.device
    tiled = torch.empty(scale_bytes(rows, K), dtype=torch.uint8, device=dev) if tiled is None else tiled
    _need(tiled, "tiled", torch.uint8, min_numel=scale_bytes(rows, K), device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_scales_to_tiled(_ptr(rowmajor), rows, K, _ptr(tiled), _stream(stream, dev)),
               "macaq_scales_to_tiled")
    return tiled


def macaq_scales_to_rowmajor(tiled: torch.Tensor, rows: int, K: int, rowmajor=None, stream=None):
    """MMA-tile-layout E8M0 scales -> row-major uint8 [rows, K/32]."""
    _need(tiled, "tiled", torch.uint8, min_numel=scale_bytes(rows, K))
    dev = tiled.device
    rowmajor = torch.empty(rows, K // 32, dtype=torch.uint8, device=dev) if rowmajor is None else rowmajor
    _need(rowmajor, "rowmajor", torch.uint8, (rows, K // 32), device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_scales_to_rowmajor(_ptr(tiled), rows, K, _ptr(rowmajor), _stream(stream, dev)),
               "macaq_scales_to_rowmajor")
    return rowmajor


def macaq_calibrate_scale(xcal: torch.Tensor, W: torch.Tensor, s=None, stream=None):
    """Per-channel scale s (fp32 [K]) from a bf16 calibration batch [C, K] and fp32 weights [N, K]."""
    C, K = xcal.shape
    _need(xcal, "xcal", torch.bfloat16)
    dev = xcal.device
    _need(W, "W", torch.float32, device=dev)
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("xcal and W must have the same K")
    s = torch.empty(K, dtype=torch.float32, device=W.device) if s is None else s
    _need(s, "s", torch.float32, (K,), device=W.device)
    with torch.cuda.device(dev):
        _check(load_library().macaq_calibrate_scale(_ptr(xcal), C, _ptr(W), N, K, _ptr(s), _stream(stream, dev)),
               "macaq_calibrate_scale")
    return s


def macaq_fold_weights(W: torch.Tensor, s: torch.Tensor, Wq=None, Ws=None, act_mult=None, stream=None):
    """Fold diag(s) H/sqrt(32) into W (fp32 [N, K]) and RTN-quantise: (Wq, Ws, act_mult)."""
    N, K = W.shape
    _need(W, "W", torch.float32)
    dev = W.device
    _need(s, "s", torch.float32, (K,), device=dev)
    Wq = torch.empty(N, K // 2, dtype=torch.uint8, device=dev) if Wq is None else Wq
    Ws = torch.empty(max(scale_bytes(N, K), 1), dtype=torch.uint8, device=dev) if Ws is None else Ws
    act_mult = torch.empty(K, dtype=torch.float32, device=dev) if act_mult is None else act_mult
    _need(Wq, "Wq", torch.uint8, (N, K // 2), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=scale_bytes(N, K), device=dev)
    _need(act_mult, "act_mult", torch.float32, (K,), device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_fold_weights(_ptr(W), N, K, _ptr(s), _ptr(Wq), _ptr(Ws), _ptr(act_mult),
                                                 _stream(stream, dev)), "macaq_fold_weights")
    return Wq, Ws, act_mult


def macaq_act_transform_quant(x: torch.Tensor, act_mult: torch.Tensor, Aq=None, As=None, stream=None):
    """Scale, FWHT-32 and MXFP4-quantise bf16 activations [M, K]: (Aq, As)."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    dev = x.device
    _need(act_mult, "act_mult", torch.float32, (K,), device=dev)
    Aq = torch.empty(M, K // 2, dtype=torch.uint8, device=dev) if Aq is None else Aq
    As = torch.empty(max(scale_bytes(M, K), 1), dtype=torch.uint8, device=dev) if As is None else As
    _need(Aq, "Aq", torch.uint8, (M, K // 2), device=dev)
    _need(As, "As", torch.uint8, min_numel=scale_bytes(M, K), device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_act_transform_quant(_ptr(x), M, K, _ptr(act_mult), _ptr(Aq), _ptr(As),
                                                        _stream(stream, dev)), "macaq_act_transform_quant")
    return Aq, As


def macaq_act_quant_plain(x: torch.Tensor, Aq=None, As=None, stream=None):
    """Plain MXFP4 quantisation of bf16 activations (no scale, no transform): (Aq, As)."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    dev = x.device
    Aq = torch.empty(M, K // 2, dtype=torch.uint8, device=dev) if Aq is None else Aq
    As = torch.empty(max(scale_bytes(M, K), 1), dtype=torch.uint8, device=dev) if As is None else As
    _need(Aq, "Aq", torch.uint8, (M, K // 2), device=dev)
    _need(As, "As", torch.uint8, min_numel=scale_bytes(M, K), device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_act_quant_plain(_ptr(x), M, K, _ptr(Aq), _ptr(As), _stream(stream, dev)),
               "macaq_act_quant_plain")
    return Aq, As


def macaq_mxfp4_gemm(Aq, As, Wq, Ws, M: int, N: int, K: int, y=None, out_fp32: bool = False, workspace=None,
                     data_parallel: bool = False, stream=None):
    """y = dec(A) dec(W)^T from MXFP4 operands; bf16 (default) or fp32 [M, N].  A stream-K
    workspace is allocated when not given (the schedule macaq_w4a4_linear uses);
    data_parallel=True passes none (data-parallel schedule)."""
    _need(Aq, "Aq", torch.uint8, (M, K // 2))
    dev = Aq.device
    _need(Wq, "Wq", torch.uint8, (N, K // 2), device=dev)
    _need(As, "As", torch.uint8, min_numel=scale_bytes(M, K), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=scale_bytes(N, K), device=dev)
    dt = torch.float32 if out_fp32 else torch.bfloat16
    y = torch.empty(M, N, dtype=dt, device=dev) if y is None else y
    _need(y, "y", dt, (M, N), device=dev)
    if data_parallel:
        workspace = None
    elif workspace is None:
        workspace = torch.empty(max(gemm_workspace_bytes(M, N, K, dev), 1), dtype=torch.uint8, device=dev)
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_mxfp4_gemm(_ptr(Aq), _ptr(As), M, _ptr(Wq), _ptr(Ws), N, K, _ptr(y),
                                               1 if out_fp32 else 0, _ptr(workspace),
                                               0 if workspace is None else workspace.numel(), _stream(stream, dev)),
               "macaq_mxfp4_gemm")
    return y


def macaq_w4a4_linear(x: torch.Tensor, act_mult: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, N: int,
                      y=None, workspace=None, stream=None):
    """y = x W^T through the online transform, MXFP4 quantisation and the W4A4 GEMM (bf16 [M, N])."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    dev = x.device
    _need(act_mult, "act_mult", torch.float32, (K,), device=dev)
    _need(Wq, "Wq", torch.uint8, (N, K // 2), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=scale_bytes(N, K), device=dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev) if y is None else y
    _need(y, "y", torch.bfloat16, (M, N), device=dev)
    need = linear_workspace_bytes(M, N, K, dev)
    workspace = torch.empty(need, dtype=torch.uint8, device=dev) if workspace is None else workspace
    _need(workspace, "workspace", torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_w4a4_linear(_ptr(x), M, K, _ptr(act_mult), _ptr(Wq), _ptr(Ws), N, _ptr(y),
                                                _ptr(workspace), workspace.numel(), _stream(stream, dev)),
               "macaq_w4a4_linear")
    return y


def macaq_mxfp4_linear(x: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, N: int, y=None, workspace=None,
                       stream=None):
    """Plain MXFP4 linear (no scale, no transform): the baseline of the transform's overhead."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    dev = x.device
    _need(Wq, "Wq", torch.uint8, (N, K // 2), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=scale_bytes(N, K), device=dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev) if y is None else y
    _need(y, "y", torch.bfloat16, (M, N), device=dev)
    need = linear_workspace_bytes(M, N, K, dev)
    workspace = torch.empty(need, dtype=torch.uint8, device=dev) if workspace is None else workspace
    _need(workspace, "workspace", torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_mxfp4_linear(_ptr(x), M, K, _ptr(Wq), _ptr(Ws), N, _ptr(y), _ptr(workspace),
                                                 workspace.numel(), _stream(stream, dev)), "macaq_mxfp4_linear")
    return y


def linear_multi_workspace_bytes(M: int, G: int, K: int, device=None) -> int:
    """Scratch bytes macaq_w4a4_linear_multi needs for G linears on M tokens (default device: the
    current one; the size depends on its SM count)."""
    with _device(device):
        return int(load_library().macaq_linear_multi_workspace_bytes(M, G, K))


def macaq_w4a4_linear_multi(x: torch.Tensor, act_mult, Wq: torch.Tensor, Ws: torch.Tensor, Ns, y=None,
                            workspace=None, stream=None):
    """G linears on the same x [M, K] bf16 (the q, k and v projections, or gate and up), each its own
    folded layer: act_mult fp32 [G, K] (torch.stack of the folds' multipliers; None: plain MXFP4),
    Wq [sum Ns, K/2] and Ws (torch.cat of the folds' codes and scales, in the same order), Ns the
    output features of each (multiples of 128).  Returns y bf16 [M, sum Ns]: linear g's outputs in
    columns sum(Ns[:g]) .. sum(Ns[:g + 1]) - 1."""
    import numpy as np
    M, K = x.shape
    n = np.ascontiguousarray(np.asarray(list(Ns), dtype=np.int64))
    G, Nt = len(n), int(n.sum())
    _need(x, "x", torch.bfloat16)
    dev = x.device
    if act_mult is not None:
        _need(act_mult, "act_mult", torch.float32, (G, K), device=dev)
    _need(Wq, "Wq", torch.uint8, (Nt, K // 2), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=sum(scale_bytes(int(v), K) for v in n), device=dev)
    y = torch.empty(M, Nt, dtype=torch.bfloat16, device=dev) if y is None else y
    _need(y, "y", torch.bfloat16, (M, Nt), device=dev)
    need = linear_multi_workspace_bytes(M, G, K, dev)
    workspace = torch.empty(need, dtype=torch.uint8, device=dev) if workspace is None else workspace
    _need(workspace, "workspace", torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_w4a4_linear_multi(_ptr(x), M, K, G, _ptr(act_mult), _ptr(Wq), _ptr(Ws),
                                                      ctypes.c_void_p(n.ctypes.data), _ptr(y), _ptr(workspace),
                                                      workspace.numel(), _stream(stream, dev)),
               "macaq_w4a4_linear_multi")
    return y


def _counts_array(counts):
    import numpy as np
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.int64))
    return c, ctypes.c_void_p(c.ctypes.data)


def grouped_workspace_bytes(counts, N: int, K: int) -> int:
    """Scratch bytes macaq_w4a4_grouped_linear needs for these per-expert token counts."""
    c, cp = _counts_array(counts)
    return int(load_library().macaq_grouped_workspace_bytes(cp, len(c), N, K))


def macaq_w4a4_grouped_linear(x: torch.Tensor, counts, act_mult, Wq: torch.Tensor, Ws: torch.Tensor, N: int,
                              y=None, workspace=None, stream=None):
    """Grouped (mixture-of-experts) linear: x [T, K] bf16 grouped by expert, counts = tokens per
    expert (host ints), act_mult fp32 [E, K] (None: plain MXFP4), Wq [E, N, K/2], Ws the experts'
    scale buffers concatenated.  Returns y bf16 [T, N]."""
    T, K = x.shape
    c, cp = _counts_array(counts)
    E = len(c)
    if int(c.sum()) != T:
        raise ValueError("counts must sum to the rows of x")
    _need(x, "x", torch.bfloat16)
    dev = x.device
    if act_mult is not None:
        _need(act_mult, "act_mult", torch.float32, (E, K), device=dev)
    _need(Wq, "Wq", torch.uint8, (E, N, K // 2), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=E * scale_bytes(N, K), device=dev)
    y = torch.empty(T, N, dtype=torch.bfloat16, device=dev) if y is None else y
    _need(y, "y", torch.bfloat16, (T, N), device=dev)
    need = max(grouped_workspace_bytes(c, N, K), 1)
    workspace = torch.empty(need, dtype=torch.uint8, device=dev) if workspace is None else workspace
    _need(workspace, "workspace", torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_w4a4_grouped_linear(_ptr(x), cp, E, K, _ptr(act_mult), _ptr(Wq), _ptr(Ws), N,
                                                        _ptr(y), _ptr(workspace), workspace.numel(), _stream(stream, dev)),
               "macaq_w4a4_grouped_linear")
    return y


def grouped_device_workspace_bytes(T: int, E: int, N: int, K: int, device=None) -> int:
    """Scratch bytes macaq_w4a4_grouped_linear_device needs for T routed rows over E experts."""
    with _device(device):
        return int(load_library().macaq_grouped_device_workspace_bytes(T, E, N, K))


def macaq_w4a4_grouped_linear_device(x: torch.Tensor, counts: torch.Tensor, act_mult, Wq: torch.Tensor,
                                     Ws: torch.Tensor, N: int, capacity: int = 0, y=None, workspace=None, stream=None):
    """Grouped (mixture-of-experts) linear with the per-expert token counts on the DEVICE (int32 or
    int64 CUDA tensor [E], e.g. straight from a GPU router): no host copy, no synchronisation.  x
    [T, K] bf16 grouped by expert, act_mult fp32 [E, K] (None: plain MXFP4), Wq [E, N, K/2], Ws the
    experts' scale buffers concatenated; capacity = the most rows any expert may have (0: T), which
    picks the kernels; rows past it are not computed (reported as MACAQ_ECOUNTS).  Returns y bf16
    [T, N]."""
    T, K = x.shape
    _need(x, "x", torch.bfloat16)
    dev = x.device
    if counts.dtype not in (torch.int32, torch.int64):
        raise ValueError("counts must be int32 or int64")
    _need(counts, "counts", counts.dtype, device=dev)
    E = counts.numel()
    if act_mult is not None:
        _need(act_mult, "act_mult", torch.float32, (E, K), device=dev)
    _need(Wq, "Wq", torch.uint8, (E, N, K // 2), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=E * scale_bytes(N, K), device=dev)
    y = torch.empty(T, N, dtype=torch.bfloat16, device=dev) if y is None else y
    _need(y, "y", torch.bfloat16, (T, N), device=dev)
    need = grouped_device_workspace_bytes(T, E, N, K, dev)
    if need == 0:
        raise ValueError("shape not supported by the grouped linear (1 <= E <= 128, N % 128 == 0, T >= 1)")
    workspace = torch.empty(need, dtype=torch.uint8, device=dev) if workspace is None else workspace
    _need(workspace, "workspace", torch.uint8, min_numel=need, device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_w4a4_grouped_linear_device(
            _ptr(x), T, _ptr(counts), counts.element_size(), E, int(capacity), K, _ptr(act_mult), _ptr(Wq), _ptr(Ws), N,
            _ptr(y),
            _ptr(workspace), workspace.numel(), _stream(stream, dev)), "macaq_w4a4_grouped_linear_device")
    return y


NOALLOC_SCRATCH_BYTES = 32 << 20  # MACAQ_NOALLOC_SCRATCH_BYTES of include/macaq.h


def macaq_w4a4_linear_noalloc(x: torch.Tensor, act_mult: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor,
                              N: int, y=None, stream=None):
    """macaq_w4a4_linear without a workspace: for callers that cannot allocate device memory,
    the library keeps the activation scratch in its own static 32 MiB device array (see
    include/macaq.h for the limit and the ordering rule).  Only y is allocated here, and
    only when the caller does not pass it."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    dev = x.device
    _need(act_mult, "act_mult", torch.float32, (K,), device=dev)
    _need(Wq, "Wq", torch.uint8, (N, K // 2), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=scale_bytes(N, K), device=dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev) if y is None else y
    _need(y, "y", torch.bfloat16, (M, N), device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_w4a4_linear_noalloc(_ptr(x), M, K, _ptr(act_mult), _ptr(Wq), _ptr(Ws), N, _ptr(y),
                                                        _stream(stream, dev)), "macaq_w4a4_linear_noalloc")
    return y


def macaq_calib_hessian(xcal: torch.Tensor, act_mult: torch.Tensor, Hs=None, workspace=None, stream=None):
    """Hs = Xt^T Xt (fp64 [K, K]) of a bf16 calibration batch [C, K] after the online transform with
    the layer's multipliers (Flip-Refinement's Hessian)."""
    C, K = xcal.shape
    _need(xcal, "xcal", torch.bfloat16)
    dev = xcal.device
    _need(act_mult, "act_mult", torch.float32, (K,), device=dev)
    Hs = torch.empty(K, K, dtype=torch.float64, device=dev) if Hs is None else Hs
    _need(Hs, "Hs", torch.float64, (K, K), device=dev)
    need = int(load_library().macaq_hessian_workspace_bytes(C, K))
    workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev) if workspace is None else workspace
    _need(workspace, "workspace", torch.uint8, min_numel=need, device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_calib_hessian(_ptr(xcal), C, K, _ptr(act_mult), _ptr(Hs), _ptr(workspace),
                                                  workspace.numel(), _stream(stream, dev)), "macaq_calib_hessian")
    return Hs


def macaq_flip_refine(W: torch.Tensor, s: torch.Tensor, Hs: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor,
                      max_moves: int, moves=None, workspace=None, stream=None):
    """Flip-Refinement of the round-to-nearest codes Wq [N, K/2] (from macaq_fold_weights of W and s)
    in place, scales Ws kept; returns the int32 moves applied per row."""
    N, K = W.shape
    _need(W, "W", torch.float32)
    dev = W.device
    _need(s, "s", torch.float32, (K,), device=dev)
    _need(Hs, "Hs", torch.float64, (K, K), device=dev)
    _need(Wq, "Wq", torch.uint8, (N, K // 2), device=dev)
    _need(Ws, "Ws", torch.uint8, min_numel=scale_bytes(N, K), device=dev)
    moves = torch.empty(N, dtype=torch.int32, device=dev) if moves is None else moves
    _need(moves, "moves", torch.int32, (N,), device=dev)
    need = int(load_library().macaq_flip_refine_workspace_bytes(N, K))
    if need == 0:
        raise ValueError(f"K={K} is not supported by macaq_flip_refine (K <= 12288, K % 32 == 0)")
    workspace = torch.empty(need, dtype=torch.uint8, device=dev) if workspace is None else workspace
    _need(workspace, "workspace", torch.uint8, min_numel=need, device=dev)
    with torch.cuda.device(dev):
        _check(load_library().macaq_flip_refine(_ptr(W), N, K, _ptr(s), _ptr(Hs), _ptr(Wq), _ptr(Ws), int(max_moves),
                                                _ptr(moves), _ptr(workspace), workspace.numel(),
                                                _stream(stream, dev)), "macaq_flip_refine")
    return moves


def macaq_device_status(clear: bool = False) -> int:
    """MACAQ_OK, or the last device-side event: MACAQ_ETIMEOUT (a bounded wait gave up) or
    MACAQ_ECOUNTS (device routing counts were corrected).  Synchronises."""
    return int(load_library().macaq_device_status(1 if clear else 0))
