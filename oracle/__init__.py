"""CPU oracle of the LLM.int8() linear layer (ctypes wrapper around oracle.c).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and bench.py's CPU
baseline / reference legs may import this module; the product package never does.
The C source restates the pages' definitions (see oracle.c for the citations and
the readings taken where the pages are silent).

All arrays are numpy; half-precision data travels as ``np.float16``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain C99, -O2, OpenMP over output rows)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-fopenmp",
            "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # INT8_ORACLE_LIB lets the mutation tests load a deliberately broken build.
            lib = ctypes.CDLL(os.environ.get("INT8_ORACLE_LIB") or build())
            i64, i32, f32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float
            p = ctypes.c_void_p
            lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_half_to_double.restype = ctypes.c_double
            lib.oracle_half_from_double.argtypes = [ctypes.c_double]
            lib.oracle_half_from_double.restype = ctypes.c_uint16
            lib.oracle_quant_weight.argtypes = [p, i64, i64, p, p]
            lib.oracle_outlier_columns.argtypes = [p, i64, i64, f32, p, p, p]
            lib.oracle_quantize_rows.argtypes = [p, i64, i64, p, p, p]
            lib.oracle_gemm_i32.argtypes = [p, p, i64, i64, i64, p]
            lib.oracle_outlier_weights.argtypes = [p, p, i64, i64, p, i32, p]
            lib.oracle_linear_forward.argtypes = [p, i64, i64, p, p, p, i64, f32, p]
            lib.oracle_linear_forward_rows.argtypes = [p, i64, i64, p, p, p, i64, f32, p, i64, p, p]
            lib.oracle_linear_forward_rows_w16.argtypes = [p, i64, i64, p, p, p, p, i64, f32, p,
                                                           i64, p, p]
            lib.oracle_quantize_tensor.argtypes = [p, i64, i64, p, p, p]
            lib.oracle_linear_forward_rows_ex.argtypes = [p, i64, i64, p, p, p, p, i64, f32,
                                                          ctypes.c_int, p, i64, p, p]
            lib.oracle_activation_stats.argtypes = [p, i64, i64, p, p]
            for name in ("oracle_quant_weight", "oracle_outlier_columns", "oracle_quantize_rows",
                         "oracle_gemm_i32", "oracle_outlier_weights", "oracle_linear_forward",
                         "oracle_linear_forward_rows", "oracle_linear_forward_rows_w16",
                         "oracle_quantize_tensor", "oracle_linear_forward_rows_ex",
                         "oracle_activation_stats"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise OracleError(f"{what} returned {rc}")


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def half_to_double(bits: int) -> float:
    return _load().oracle_half_to_double(int(bits))


def half_from_double(x: float) -> int:
    return int(_load().oracle_half_from_double(float(x)))


def quant_weight(W):
    W = _c(W, np.float16)
    N, K = W.shape
    Wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    _check(_load().oracle_quant_weight(_ptr(W), N, K, _ptr(Wq), _ptr(sw)), "oracle_quant_weight")
    return Wq, sw


def outlier_columns(X, threshold: float):
    X = _c(X, np.float16)
    M, K = X.shape
    mask = np.empty((K + 31) // 32, np.uint32)
    cols = np.empty(K, np.int32)
    n = np.zeros(1, np.int32)
    _check(_load().oracle_outlier_columns(_ptr(X), M, K, float(threshold), _ptr(mask), _ptr(cols),
                                          _ptr(n)), "oracle_outlier_columns")
    return mask, cols[: int(n[0])].copy()


def quantize_rows(X, mask):
    X = _c(X, np.float16)
    mask = _c(mask, np.uint32)
    M, K = X.shape
    Xq = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    _check(_load().oracle_quantize_rows(_ptr(X), M, K, _ptr(mask), _ptr(Xq), _ptr(sx)),
           "oracle_quantize_rows")
    return Xq, sx


def gemm_i32(Xq, Wq):
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = Xq.shape
    N = Wq.shape[0]
    A = np.empty((M, N), np.int32)
    _check(_load().oracle_gemm_i32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(A)), "oracle_gemm_i32")
    return A


def outlier_weights(Wq, sw, cols):
    Wq = _c(Wq, np.int8)
    sw = _c(sw, np.float32)
    cols = _c(cols, np.int32)
    N, K = Wq.shape
    W_hat = np.empty((N, len(cols)), np.float16)
    _check(_load().oracle_outlier_weights(_ptr(Wq), _ptr(sw), N, K, _ptr(cols), len(cols),
                                          _ptr(W_hat)), "oracle_outlier_weights")
    return W_hat


def linear_forward(X, Wq, sw, bias, threshold: float):
    X = _c(X, np.float16)
    Wq = _c(Wq, np.int8)
    sw = _c(sw, np.float32)
    b = None if bias is None else _c(bias, np.float16)
    M, K = X.shape
    N = Wq.shape[0]
    Y = np.empty((M, N), np.float16)
    _check(_load().oracle_linear_forward(_ptr(X), M, K, _ptr(Wq), _ptr(sw), _ptr(b), N,
                                         float(threshold), _ptr(Y)), "oracle_linear_forward")
    return Y


def linear_forward_rows_w16(X, Wq, sw, W16, bias, threshold: float, rows):
    """As linear_forward_rows, with the outlier columns' weights taken from the kept fp16
    weights W16 (has_fp16_weights=True)."""
    X = _c(X, np.float16)
    Wq = _c(Wq, np.int8)
    sw = _c(sw, np.float32)
    W16 = _c(W16, np.float16)
    b = None if bias is None else _c(bias, np.float16)
    rows = _c(rows, np.int64)
    M, K = X.shape
    N = Wq.shape[0]
    Y = np.empty((len(rows), N), np.float16)
    A = np.empty((len(rows), N), np.int32)
    _check(_load().oracle_linear_forward_rows_w16(_ptr(X), M, K, _ptr(Wq), _ptr(sw), _ptr(W16),
                                                  _ptr(b), N, float(threshold), _ptr(rows),
                                                  len(rows), _ptr(Y), _ptr(A)),
           "oracle_linear_forward_rows_w16")
    return Y, A


def linear_forward_w16(X, Wq, sw, W16, bias, threshold: float):
    return linear_forward_rows_w16(X, Wq, sw, W16, bias, threshold, np.arange(X.shape[0]))[0]


def linear_forward_rows(X, Wq, sw, bias, threshold: float, rows):
    """Y and the int32 accumulators of the listed rows only (outliers found over all rows)."""
    X = _c(X, np.float16)
    Wq = _c(Wq, np.int8)
    sw = _c(sw, np.float32)
    b = None if bias is None else _c(bias, np.float16)
    rows = _c(rows, np.int64)
    M, K = X.shape
    N = Wq.shape[0]
    Y = np.empty((len(rows), N), np.float16)
    A = np.empty((len(rows), N), np.int32)
    _check(_load().oracle_linear_forward_rows(_ptr(X), M, K, _ptr(Wq), _ptr(sw), _ptr(b), N,
                                              float(threshold), _ptr(rows), len(rows), _ptr(Y),
                                              _ptr(A)), "oracle_linear_forward_rows")
    return Y, A


def quantize_tensor(X, mask):
    """One activation scale for the whole of X ([P5] item 2 as its snippet is written): absmax
    over every row and the regular columns, / 127.  Returns Xq and the scale of every row (all
    equal)."""
    X = _c(X, np.float16)
    mask = _c(mask, np.uint32)
    M, K = X.shape
    Xq = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    _check(_load().oracle_quantize_tensor(_ptr(X), M, K, _ptr(mask), _ptr(Xq), _ptr(sx)),
           "oracle_quantize_tensor")
    return Xq, sx


def linear_forward_rows_ex(X, Wq, sw, bias, threshold: float, rows, W16=None,
                           per_tensor: bool = False):
    """linear_forward_rows with the kept fp16 weights (W16, nullable) and the per-tensor
    activation scale as options."""
    X = _c(X, np.float16)
    Wq = _c(Wq, np.int8)
    sw = _c(sw, np.float32)
    W16 = None if W16 is None else _c(W16, np.float16)
    b = None if bias is None else _c(bias, np.float16)
    rows = _c(rows, np.int64)
    M, K = X.shape
    N = Wq.shape[0]
    Y = np.empty((len(rows), N), np.float16)
    A = np.empty((len(rows), N), np.int32)
    _check(_load().oracle_linear_forward_rows_ex(_ptr(X), M, K, _ptr(Wq), _ptr(sw), _ptr(W16),
                                                 _ptr(b), N, float(threshold), int(per_tensor),
                                                 _ptr(rows), len(rows), _ptr(Y), _ptr(A)),
           "oracle_linear_forward_rows_ex")
    return Y, A


def linear_forward_tensor(X, Wq, sw, bias, threshold: float, W16=None):
    """The layer with one activation scale for the whole of X."""
    return linear_forward_rows_ex(X, Wq, sw, bias, threshold, np.arange(X.shape[0]), W16=W16,
                                  per_tensor=True)[0]


def activation_stats(X):
    """[P2] section 5.1: (max |X|, the 0.99 quantile of |X|, max / (q99 + 1e-6), column
    absmax [K])."""
    X = _c(X, np.float16)
    M, K = X.shape
    col = np.empty(K, np.float32)
    out = np.empty(3, np.float64)
    _check(_load().oracle_activation_stats(_ptr(X), M, K, _ptr(col), _ptr(out)),
           "oracle_activation_stats")
    return float(out[0]), float(out[1]), float(out[2]), col

