"""CPU oracle for the MACaQ W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path (``online_hadamard_b200``) never does, and the two
share no code: this package wraps ``macaq_oracle.c`` (plain C, built with gcc on first
use) with numpy marshalling and nothing else.

Every function follows "MACaQ: Fast, Model Agnostic Calibrated Quantization for
Low-Precision Weights and Activations", Abstract (per-channel scale and block-Hadamard
applied online to activations, inverse transforms absorbed into the weights, MXFP4 W4A4,
round-to-nearest weights), with the readings stated at the top of ``macaq_oracle.c``.

Parity pins (tests/test_oracle_pins.py) tie every function here to something other than
itself: the Sylvester matrix built from its popcount definition, closed forms, scale and
sign invariants, brute-force nearest-value search, a hand-derived worked case
(tests/golden/) and an exact fp64 contraction.  The only unpinned quantity is the
end-to-end quantisation error against the unquantised product, which the pages do not
bound ("parity unpinned"; it is reported, not gated).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "macaq_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libmacaq_oracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile macaq_oracle.c into _build/libmacaq_oracle.so (gcc, IEEE fp32/fp64)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            p = ctypes.c_void_p
            i64 = ctypes.c_int64
            lib.oracle_multipliers.argtypes = [p, i64, p, p]
            lib.oracle_transform_f32.argtypes = [p, i64, i64, p, p]
            lib.oracle_transform_f64.argtypes = [p, i64, i64, p, p]
            lib.oracle_e8m0_from_amax.argtypes = [ctypes.c_float]
            lib.oracle_e8m0_from_amax.restype = ctypes.c_int
            lib.oracle_e2m1_index.argtypes = [ctypes.c_double]
            lib.oracle_e2m1_index.restype = ctypes.c_int
            lib.oracle_e2m1_code.argtypes = [ctypes.c_float, ctypes.c_int]
            lib.oracle_e2m1_code.restype = ctypes.c_int
            lib.oracle_quantize_mx.argtypes = [p, i64, i64, p, p]
            lib.oracle_act_transform_quant.argtypes = [p, i64, i64, p, p, p]
            lib.oracle_fold_weights.argtypes = [p, i64, i64, p, p, p, p]
            lib.oracle_mx_decode.argtypes = [p, p, i64, i64, p]
            lib.oracle_mx_gemm.argtypes = [p, p, p, i64, p, p, i64, i64, p]
            lib.oracle_calibrate_scale.argtypes = [p, i64, p, i64, i64, p]
            lib.oracle_hessian.argtypes = [p, i64, i64, p]
            lib.oracle_flip_refine.argtypes = [p, i64, i64, p, p, p, i64, p]
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _check_k(K: int) -> None:
    if K % 32:
        raise ValueError(f"K={K} is not a multiple of the 32-element block")


def multipliers(s) -> tuple[np.ndarray, np.ndarray]:
    """(act_mult, w_mult) = (fl32(c/s_k), fl32(s_k*c)), c = 1/sqrt(32) in fp64."""
    s = _f32(s)
    a = np.empty_like(s)
    w = np.empty_like(s)
    _load().oracle_multipliers(_ptr(s), s.size, _ptr(a), _ptr(w))
    return a, w


def transform_f32(X, mult) -> np.ndarray:
    """u = fl32(x * mult) per channel, then the unnormalised FWHT-32 per block (fp32)."""
    X = _f32(X)
    R, K = X.shape
    _check_k(K)
    mult = _f32(mult)
    V = np.empty_like(X)
    _load().oracle_transform_f32(_ptr(X), R, K, _ptr(mult), _ptr(V))
    return V


def transform_f64(X, mult) -> np.ndarray:
    """The scale + block-Hadamard transform in fp64 (algebra checks only)."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    R, K = X.shape
    _check_k(K)
    mult = np.ascontiguousarray(mult, dtype=np.float64)
    V = np.empty_like(X)
    _load().oracle_transform_f64(_ptr(X), R, K, _ptr(mult), _ptr(V))
    return V


def e8m0_from_amax(amax: float) -> int:
    return _load().oracle_e8m0_from_amax(float(amax))


def e2m1_index(t: float) -> int:
    return _load().oracle_e2m1_index(float(t))


def e2m1_code(v: float, e: int) -> int:
    return _load().oracle_e2m1_code(float(v), int(e))


def quantize_mx(V) -> tuple[np.ndarray, np.ndarray]:
    """MXFP4 along K: codes uint8 [R][K/2] (even k low nibble), E8M0 scales uint8 [R][K/32]."""
    V = _f32(V)
    R, K = V.shape
    _check_k(K)
    codes = np.empty((R, K // 2), np.uint8)
    scales = np.empty((R, K // 32), np.uint8)
    _load().oracle_quantize_mx(_ptr(V), R, K, _ptr(codes), _ptr(scales))
    return codes, scales


def act_transform_quant(X, act_mult) -> tuple[np.ndarray, np.ndarray]:
    """Activation path: per-channel scale, block-Hadamard b=32, MXFP4."""
    X = _f32(X)
    R, K = X.shape
    _check_k(K)
    act_mult = _f32(act_mult)
    codes = np.empty((R, K // 2), np.uint8)
    scales = np.empty((R, K // 32), np.uint8)
    _load().oracle_act_transform_quant(_ptr(X), R, K, _ptr(act_mult), _ptr(codes), _ptr(scales))
    return codes, scales


def act_quant_plain(X) -> tuple[np.ndarray, np.ndarray]:
    """Plain MXFP4 quantisation of activations (no scale, no transform)."""
    return quantize_mx(X)


def fold_weights(W, s) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Fold diag(s) H/sqrt(32) into W and RTN-quantise: (codes, scales, act_mult)."""
    W = _f32(W)
    N, K = W.shape
    _check_k(K)
    s = _f32(s)
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // 32), np.uint8)
    act_mult = np.empty(K, np.float32)
    _load().oracle_fold_weights(_ptr(W), N, K, _ptr(s), _ptr(codes), _ptr(scales), _ptr(act_mult))
    return codes, scales, act_mult


def mx_decode(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, K2 = codes.shape
    out = np.empty((R, 2 * K2), np.float64)
    _load().oracle_mx_decode(_ptr(codes), _ptr(scales), R, 2 * K2, _ptr(out))
    return out


def mx_gemm(Aq, As, Wq, Ws, rows=None) -> np.ndarray:
    """y[i][n] = sum_k dec(A)[rows[i]][k] * dec(W)[n][k], exact fp64 contraction."""
    Aq = np.ascontiguousarray(Aq, dtype=np.uint8)
    As = np.ascontiguousarray(As, dtype=np.uint8)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    Ws = np.ascontiguousarray(Ws, dtype=np.uint8)
    M, K2 = Aq.shape
    N = Wq.shape[0]
    K = 2 * K2
    if rows is None:
        rows_arr = None
        n_rows = M
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.size
        if n_rows and (rows_arr.min() < 0 or rows_arr.max() >= M):
            raise IndexError("row index out of range")
    y = np.empty((n_rows, N), np.float64)
    _load().oracle_mx_gemm(_ptr(Aq), _ptr(As), None if rows_arr is None else _ptr(rows_arr), n_rows,
                           _ptr(Wq), _ptr(Ws), N, K, _ptr(y))
    return y


def calibrate_scale(xcal, W) -> np.ndarray:
    """Per-channel scale s [K] from calibration activations xcal [C, K] and weights W [N, K]:
    fl32(sqrt(max|xcal_:,j| / max|W_:,j|)) in double, 1 where either maximum is 0."""
    xcal = _f32(xcal)
    W = _f32(W)
    C, K = xcal.shape
    N, K2 = W.shape
    if K2 != K:
        raise ValueError("xcal and W must have the same K")
    s = np.empty(K, np.float32)
    _load().oracle_calibrate_scale(_ptr(xcal), C, _ptr(W), N, K, _ptr(s))
    return s


def hessian_of(Xt) -> np.ndarray:
    """Hs = Xt^T Xt (fp64 [K][K]) of transformed calibration activations Xt [C][K] (fp32),
    each entry an fma chain over the calibration rows in order (Flip-Refinement)."""
    Xt = _f32(Xt)
    C, K = Xt.shape
    Hs = np.empty((K, K), np.float64)
    _load().oracle_hessian(_ptr(Xt), C, K, _ptr(Hs))
    return Hs


def calib_hessian(xcal, act_mult) -> np.ndarray:
    """Hs of a calibration batch xcal [C][K] (bf16 values): the online transform with the layer's
    activation multipliers, then Xt^T Xt in fp64."""
    return hessian_of(transform_f32(xcal, act_mult))


def flip_refine_codes(V, codes, scales, Hs, max_moves) -> tuple[np.ndarray, np.ndarray]:
    """Flip-Refinement (see macaq_oracle.c) of round-to-nearest codes [N][K/2] of the folded
    weights V [N][K] (fp32) with their E8M0 scales [N][K/32] kept: (refined codes, moves per row)."""
    V = _f32(V)
    N, K = V.shape
    _check_k(K)
    out = np.array(codes, dtype=np.uint8, copy=True, order="C")
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    Hs = np.ascontiguousarray(Hs, dtype=np.float64)
    if Hs.shape != (K, K) or out.shape != (N, K // 2) or scales.shape != (N, K // 32):
        raise ValueError("shape mismatch")
    moves = np.empty(N, np.int64)
    _load().oracle_flip_refine(_ptr(V), N, K, _ptr(Hs), _ptr(out), _ptr(scales), int(max_moves), _ptr(moves))
    return out, moves


def flip_refine(W, s, xcal, max_moves) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The whole offline step for one layer: fold W with s (round-to-nearest codes), Hessian of the
    transformed calibration batch, Flip-Refinement.  Returns (codes, scales, moves per row)."""
    a, w = multipliers(s)
    V = transform_f32(W, w)
    codes, scales = quantize_mx(V)
    Hs = calib_hessian(xcal, a)
    refined, moves = flip_refine_codes(V, codes, scales, Hs, max_moves)
    return refined, scales, moves


def num_threads() -> int:
    return _load().oracle_num_threads()
