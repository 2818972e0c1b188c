"""B200 (sm_100a) LLM.int8() linear layer: a thin Python binding over libint8mm.so.

Every computation runs in the library's CUDA kernels; this module only marshals torch
tensors (device memory and the current stream) into the C ABI of include/int8mm.h and
raises on a nonzero status.  There is no CPU fallback: if the library has not been
built, importing the binding's functions raises.

Functions keep the C names:
    int8_quant_weight, int8_linear_workspace_size, int8_linear_forward,
    int8_quantize_rows, int8_gemm_i32, int8_outlier_weights, int8_read_device_status,
    int8_status_string, int8_linear_forward_noalloc
and ``Int8Linear`` bundles them the way the pages use the layer
(``Linear8bitLt(in, out, bias, has_fp16_weights=False, threshold=6.0)``).
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

__all__ = [
    "Int8mmError", "load_library", "library_path",
    "int8_quant_weight", "int8_linear_workspace_size", "int8_linear_forward",
    "int8_linear_quantize", "int8_linear_matmul", "int8_linear_forward_acc",
    "int8_quantize_rows", "int8_gemm_i32", "int8_outlier_weights",
    "int8_read_device_status", "int8_status_string", "int8_linear_forward_noalloc",
    "int8_linear_forward_fp16w", "int8_linear_forward_ex", "PER_TENSOR_SCALE",
    "int8_activation_stats", "Int8Linear", "DEFAULT_THRESHOLD", "int8_linear_forward_trace",
    "int8_outlier_row", "PAIR_TILES",
]

DEFAULT_THRESHOLD = 6.0
PER_TENSOR_SCALE = 1  # int8_linear_forward_ex flag: one activation scale for the whole of X
PAIR_TILES = 2        # int8_linear_forward_ex flag: M > 128 products on CTA pairs (256 x 256)
_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libint8mm.so")
_lib = None
_lock = threading.Lock()


class Int8mmError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: status {status} ({int8_status_string(status)})")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libint8mm.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m int8_mixed_precision_absmax_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        p, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.int8_status_string.argtypes = [i]
        lib.int8_status_string.restype = ctypes.c_char_p
        lib.int8_quant_weight.argtypes = [p, i, i, p, p, p]
        lib.int8_linear_workspace_size.argtypes = [i, i, i]
        lib.int8_linear_workspace_size.restype = sz
        lib.int8_linear_forward.argtypes = [p, i, i, p, p, p, i, f, p, p, sz, p]
        lib.int8_linear_quantize.argtypes = [p, i, i, p, p, i, f, p, sz, p]
        lib.int8_linear_matmul.argtypes = [p, i, i, p, p, p, i, f, p, p, sz, p]
        lib.int8_linear_forward_acc.argtypes = [p, i, i, p, p, p, i, f, p, p, p, sz, p]
        lib.int8_quantize_rows.argtypes = [p, i, i, f, p, p, p, p, p, sz, p]
        lib.int8_gemm_i32.argtypes = [p, p, i, i, i, p, p, p]
        lib.int8_outlier_weights.argtypes = [p, p, i, i, p, p, p, p]
        lib.int8_read_device_status.argtypes = [p, p]
        lib.int8_linear_forward_noalloc.argtypes = [p, i, i, p, p, p, i, f, p, p, p]
        lib.int8_linear_forward_fp16w.argtypes = [p, i, i, p, p, p, p, i, f, p, p, sz, p]
        lib.int8_linear_forward_ex.argtypes = [p, i, i, p, p, p, p, i, f, ctypes.c_uint, p, p,
                                               p, sz, p]
        lib.int8_linear_forward_trace.argtypes = [p, i, i, p, p, p, p, i, f, ctypes.c_uint, p,
                                                  p, p, p, p, p, p, p, sz, p]
        lib.int8_activation_stats_workspace_size.argtypes = []
        lib.int8_activation_stats_workspace_size.restype = sz
        lib.int8_activation_stats.argtypes = [p, i, i, p, p, p, sz, p]
        lib.int8_outlier_row.argtypes = [p, i, f, p, p]
        for name in ("int8_quant_weight", "int8_linear_forward", "int8_linear_quantize",
                     "int8_linear_matmul", "int8_linear_forward_acc", "int8_quantize_rows",
                     "int8_gemm_i32", "int8_outlier_weights", "int8_read_device_status",
                     "int8_linear_forward_noalloc", "int8_linear_forward_fp16w",
                     "int8_linear_forward_ex", "int8_activation_stats",
                     "int8_linear_forward_trace", "int8_outlier_row"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def int8_status_string(status: int) -> str:
    return load_library().int8_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise Int8mmError(status, what)


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, dims: int | None = None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dimensions")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def int8_linear_workspace_size(M: int, N: int, K: int) -> int:
    return int(load_library().int8_linear_workspace_size(M, N, K))


def new_workspace(M: int, N: int, K: int, device) -> torch.Tensor:
    """A zeroed workspace tensor (uint8) for an [M,K] x [N,K]^T layer."""
    n = int8_linear_workspace_size(M, N, K)
    if n == 0:
        raise ValueError(f"unsupported layer shape M={M} N={N} K={K}")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def int8_quant_weight(W: torch.Tensor, Wq: torch.Tensor | None = None,
                      w_scale: torch.Tensor | None = None, stream=None):
    """Per-output-channel int8 weights and float32 scales of an fp16 [N, K] weight."""
    _need(W, torch.float16, "W", 2)
    N, K = W.shape
    if Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=W.device)
    _need(Wq, torch.int8, "Wq", 2)
    _need(w_scale, torch.float32, "w_scale", 1)
    _check(load_library().int8_quant_weight(_ptr(W), N, K, _ptr(Wq), _ptr(w_scale),
                                            ctypes.c_void_p(_stream(stream, W.device))),
           "int8_quant_weight")
    return Wq, w_scale


def int8_linear_forward(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                        bias: torch.Tensor | None, threshold: float = DEFAULT_THRESHOLD,
                        Y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """Y = LLM.int8()(X, Wq, w_scale, bias, threshold), fp16 [M, N]."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.int8, "Wq", 2)
    _need(w_scale, torch.float32, "w_scale", 1)
    M, K = X.shape
    N = Wq.shape[0]
    if bias is not None:
        _need(bias, torch.float16, "bias", 1)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, "Y", 2)
    if workspace is None:
        # a shape the library rejects gets a token buffer so the C call reports the status
        n = int8_linear_workspace_size(M, N, K)
        workspace = torch.zeros(max(n, 256), dtype=torch.uint8, device=X.device)
    _need(workspace, torch.uint8, "workspace", 1)
    _check(load_library().int8_linear_forward(
        _ptr(X), M, K, _ptr(Wq), _ptr(w_scale), _ptr(bias), N, float(threshold), _ptr(Y),
        _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream, X.device))),
        "int8_linear_forward")
    return Y


def int8_linear_forward_fp16w(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                              W16: torch.Tensor, bias: torch.Tensor | None,
                              threshold: float = DEFAULT_THRESHOLD, Y: torch.Tensor | None = None,
                              workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """int8_linear_forward for a layer that keeps its fp16 weights W16 [N, K]: the outlier
    columns are multiplied by W16 itself rather than by fp16(Wq * w_scale)."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.int8, "Wq", 2)
    _need(w_scale, torch.float32, "w_scale", 1)
    _need(W16, torch.float16, "W16", 2)
    M, K = X.shape
    N = Wq.shape[0]
    if tuple(W16.shape) != (N, K):
        raise ValueError(f"W16 must be [{N}, {K}], got {tuple(W16.shape)}")
    if bias is not None:
        _need(bias, torch.float16, "bias", 1)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, "Y", 2)
    if workspace is None:
        n = int8_linear_workspace_size(M, N, K)
        workspace = torch.zeros(max(n, 256), dtype=torch.uint8, device=X.device)
    _need(workspace, torch.uint8, "workspace", 1)
    _check(load_library().int8_linear_forward_fp16w(
        _ptr(X), M, K, _ptr(Wq), _ptr(w_scale), _ptr(W16), _ptr(bias), N, float(threshold),
        _ptr(Y), _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream, X.device))),
        "int8_linear_forward_fp16w")
    return Y


def int8_linear_forward_ex(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                           bias: torch.Tensor | None, threshold: float = DEFAULT_THRESHOLD,
                           W16: torch.Tensor | None = None, per_tensor: bool = False,
                           Y: torch.Tensor | None = None, acc: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None, stream=None,
                           pair_tiles: bool = False) -> torch.Tensor:
    """The layer with every option: the kept fp16 weights W16 (or None), one activation scale
    for the whole of X (per_tensor), the int32 accumulators written to acc (or not), and the
    products on CTA pairs (pair_tiles, for M > 128)."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.int8, "Wq", 2)
    _need(w_scale, torch.float32, "w_scale", 1)
    M, K = X.shape
    N = Wq.shape[0]
    if W16 is not None:
        _need(W16, torch.float16, "W16", 2)
        if tuple(W16.shape) != (N, K):
            raise ValueError(f"W16 must be [{N}, {K}], got {tuple(W16.shape)}")
    if bias is not None:
        _need(bias, torch.float16, "bias", 1)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, "Y", 2)
    if acc is not None:
        _need(acc, torch.int32, "acc", 2)
    if workspace is None:
        n = int8_linear_workspace_size(M, N, K)
        workspace = torch.zeros(max(n, 256), dtype=torch.uint8, device=X.device)
    _need(workspace, torch.uint8, "workspace", 1)
    flags = (PER_TENSOR_SCALE if per_tensor else 0) | (PAIR_TILES if pair_tiles else 0)
    _check(load_library().int8_linear_forward_ex(
        _ptr(X), M, K, _ptr(Wq), _ptr(w_scale), _ptr(W16), _ptr(bias), N, float(threshold),
        flags, _ptr(Y), _ptr(acc), _ptr(workspace), workspace.numel(),
        ctypes.c_void_p(_stream(stream, X.device))), "int8_linear_forward_ex")
    return Y


def int8_linear_forward_trace(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                              bias: torch.Tensor | None, threshold: float = DEFAULT_THRESHOLD,
                              W16: torch.Tensor | None = None, per_tensor: bool = False,
                              workspace: torch.Tensor | None = None, stream=None,
                              pair_tiles: bool = False) -> dict:
    """One forward that also returns what its own kernels computed on the way: a dict of
    device tensors Y [M,N] fp16, acc [M,N] int32, Xq [M,K] int8, row_scale [M] f32,
    outlier_cols [K] i32 (first n_outliers valid), n_outliers [1] i32 and W_hat [N,K] fp16
    (valid at the outlier columns; zero elsewhere)."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.int8, "Wq", 2)
    _need(w_scale, torch.float32, "w_scale", 1)
    M, K = X.shape
    N = Wq.shape[0]
    dev = X.device
    if W16 is not None:
        _need(W16, torch.float16, "W16", 2)
        if tuple(W16.shape) != (N, K):
            raise ValueError(f"W16 must be [{N}, {K}], got {tuple(W16.shape)}")
    if bias is not None:
        _need(bias, torch.float16, "bias", 1)
    out = {"Y": torch.empty((M, N), dtype=torch.float16, device=dev),
           "acc": torch.empty((M, N), dtype=torch.int32, device=dev),
           "Xq": torch.empty((M, K), dtype=torch.int8, device=dev),
           "row_scale": torch.empty(M, dtype=torch.float32, device=dev),
           "outlier_cols": torch.empty(K, dtype=torch.int32, device=dev),
           "n_outliers": torch.zeros(1, dtype=torch.int32, device=dev),
           "W_hat": torch.zeros((N, K), dtype=torch.float16, device=dev)}
    if workspace is None:
        workspace = new_workspace(M, N, K, dev)
    _need(workspace, torch.uint8, "workspace", 1)
    flags = (PER_TENSOR_SCALE if per_tensor else 0) | (PAIR_TILES if pair_tiles else 0)
    _check(load_library().int8_linear_forward_trace(
        _ptr(X), M, K, _ptr(Wq), _ptr(w_scale), _ptr(W16), _ptr(bias), N, float(threshold),
        flags, _ptr(out["Y"]), _ptr(out["acc"]), _ptr(out["Xq"]), _ptr(out["row_scale"]),
        _ptr(out["outlier_cols"]), _ptr(out["n_outliers"]), _ptr(out["W_hat"]),
        _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream, dev))),
        "int8_linear_forward_trace")
    return out


def int8_activation_stats(X: torch.Tensor, stream=None):
    """Statistics of |X| for choosing the threshold: (max, q99, max / (q99 + 1e-6)) as a
    float64 tensor of 3 on the device, and the column absmax [K] (float32)."""
    _need(X, torch.float16, "X", 2)
    M, K = X.shape
    out = torch.empty(3, dtype=torch.float64, device=X.device)
    col = torch.empty(K, dtype=torch.float32, device=X.device)
    ws = torch.empty(int(load_library().int8_activation_stats_workspace_size()),
                     dtype=torch.uint8, device=X.device)
    _check(load_library().int8_activation_stats(
        _ptr(X), M, K, _ptr(col), _ptr(out), _ptr(ws), ws.numel(),
        ctypes.c_void_p(_stream(stream, X.device))), "int8_activation_stats")
    return out, col


def int8_outlier_row(col_absmax: torch.Tensor, threshold: float, row: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """fp16 [K]: col_absmax[j] where it exceeds the threshold, 0 elsewhere (the extra row the
    token split appends so that every rank finds the global outlier columns)."""
    _need(col_absmax, torch.float32, "col_absmax", 1)
    K = col_absmax.shape[0]
    if row is None:
        row = torch.empty(K, dtype=torch.float16, device=col_absmax.device)
    _need(row, torch.float16, "row", 1)
    _check(load_library().int8_outlier_row(_ptr(col_absmax), K, float(threshold), _ptr(row),
                                           ctypes.c_void_p(_stream(stream, col_absmax.device))),
           "int8_outlier_row")
    return row


def int8_linear_forward_noalloc(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                                bias: torch.Tensor | None, threshold: float, Y: torch.Tensor,
                                dev_status: torch.Tensor | None = None,
                                stream=None) -> torch.Tensor:
    """int8_linear_forward for M <= 16 with no workspace argument.

    For callers that cannot allocate device memory where they run the layer (a stream being
    captured, an allocator that must not grow): the library keeps the scratch in a static
    device array, so nothing here allocates -- Y (and dev_status, an optional int32 that
    receives a device-side failure code) come from the caller.  Calls that overlap on the
    GPU share that array and race; keep them on one stream."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.int8, "Wq", 2)
    _need(w_scale, torch.float32, "w_scale", 1)
    _need(Y, torch.float16, "Y", 2)
    if bias is not None:
        _need(bias, torch.float16, "bias", 1)
    if dev_status is not None:
        _need(dev_status, torch.int32, "dev_status", 1)
    M, K = X.shape
    _check(load_library().int8_linear_forward_noalloc(
        _ptr(X), M, K, _ptr(Wq), _ptr(w_scale), _ptr(bias), Wq.shape[0], float(threshold),
        _ptr(Y), _ptr(dev_status), ctypes.c_void_p(_stream(stream, X.device))),
        "int8_linear_forward_noalloc")
    return Y


def int8_linear_quantize(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                         threshold: float, workspace: torch.Tensor, stream=None) -> None:
    """The activation side of the forward, into `workspace` (see int8_linear_forward)."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.int8, "Wq", 2)
    _need(workspace, torch.uint8, "workspace", 1)
    M, K = X.shape
    _check(load_library().int8_linear_quantize(
        _ptr(X), M, K, _ptr(Wq), _ptr(w_scale), Wq.shape[0], float(threshold), _ptr(workspace),
        workspace.numel(), ctypes.c_void_p(_stream(stream, X.device))), "int8_linear_quantize")


def int8_linear_matmul(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                       bias: torch.Tensor | None, threshold: float, Y: torch.Tensor,
                       workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """The second half of the forward, from `workspace` (see int8_linear_forward)."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.int8, "Wq", 2)
    _need(Y, torch.float16, "Y", 2)
    _need(workspace, torch.uint8, "workspace", 1)
    M, K = X.shape
    N = Wq.shape[0]
    _check(load_library().int8_linear_matmul(
        _ptr(X), M, K, _ptr(Wq), _ptr(w_scale), _ptr(bias), N, float(threshold), _ptr(Y),
        _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream, X.device))),
        "int8_linear_matmul")
    return Y


def int8_linear_forward_acc(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                            bias: torch.Tensor | None, threshold: float = DEFAULT_THRESHOLD,
                            workspace: torch.Tensor | None = None, stream=None):
    """(Y fp16 [M,N], int32 accumulators [M,N]) of one forward."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.int8, "Wq", 2)
    M, K = X.shape
    N = Wq.shape[0]
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=X.device)
    if workspace is None:
        workspace = new_workspace(M, N, K, X.device)
    _check(load_library().int8_linear_forward_acc(
        _ptr(X), M, K, _ptr(Wq), _ptr(w_scale), _ptr(bias), N, float(threshold), _ptr(Y),
        _ptr(acc), _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream, X.device))),
        "int8_linear_forward_acc")
    return Y, acc


def int8_quantize_rows(X: torch.Tensor, threshold: float = DEFAULT_THRESHOLD,
                       workspace: torch.Tensor | None = None, stream=None):
    """(Xq int8 [M,K], row_scale f32 [M], outlier_cols i32 [K], n_outliers i32 [1]) on device.

    Only the first n_outliers entries of outlier_cols are meaningful."""
    _need(X, torch.float16, "X", 2)
    M, K = X.shape
    dev = X.device
    Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    sx = torch.empty(M, dtype=torch.float32, device=dev)
    cols = torch.empty(K, dtype=torch.int32, device=dev)
    n = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = new_workspace(M, 1, K, dev)
    _check(load_library().int8_quantize_rows(
        _ptr(X), M, K, float(threshold), _ptr(Xq), _ptr(sx), _ptr(cols), _ptr(n),
        _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream, dev))),
        "int8_quantize_rows")
    return Xq, sx, cols, n


def int8_gemm_i32(Xq: torch.Tensor, Wq: torch.Tensor, C: torch.Tensor | None = None,
                  dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """C = Xq . Wq^T exactly, int32 [M, N], on the tensor cores."""
    _need(Xq, torch.int8, "Xq", 2)
    _need(Wq, torch.int8, "Wq", 2)
    M, K = Xq.shape
    N = Wq.shape[0]
    if C is None:
        C = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=Xq.device)
    _check(load_library().int8_gemm_i32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(C), _ptr(dev_status),
                                        ctypes.c_void_p(_stream(stream, Xq.device))),
           "int8_gemm_i32")
    return C


def int8_outlier_weights(Wq: torch.Tensor, w_scale: torch.Tensor, cols: torch.Tensor,
                         n_outliers: torch.Tensor, W_hat: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """fp16 [N, K] whose first n_outliers columns are fp16(Wq[:, cols] * w_scale)."""
    _need(Wq, torch.int8, "Wq", 2)
    N, K = Wq.shape
    if W_hat is None:
        W_hat = torch.zeros((N, K), dtype=torch.float16, device=Wq.device)
    _check(load_library().int8_outlier_weights(
        _ptr(Wq), _ptr(w_scale), N, K, _ptr(cols), _ptr(n_outliers), _ptr(W_hat),
        ctypes.c_void_p(_stream(stream, Wq.device))), "int8_outlier_weights")
    return W_hat


def int8_read_device_status(dev_status: torch.Tensor, stream=None) -> int:
    """Wait for the stream and return the device status word (0 or a negative code)."""
    return int(load_library().int8_read_device_status(
        _ptr(dev_status), ctypes.c_void_p(_stream(stream, dev_status.device))))


class Int8Linear:
    """An LLM.int8() linear layer.

    Mirrors ``Linear8bitLt(in_features, out_features, bias, has_fp16_weights, threshold)``:
    the fp16 weight is quantized once per output channel at construction, then every call
    quantizes its activations per row on the fly and routes the columns whose magnitude
    exceeds ``threshold`` through fp16.  With ``has_fp16_weights=False`` (the default) only
    the int8 weights are kept and the outlier columns use fp16(Wq * w_scale); with True the
    layer also keeps the fp16 weight and the outlier columns use it.  With
    ``per_tensor_activation=True`` one activation scale serves the whole input (the default is
    one per row).
    """

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None = None,
                 threshold: float = DEFAULT_THRESHOLD, has_fp16_weights: bool = False,
                 per_tensor_activation: bool = False):
        if math.isnan(threshold):
            raise ValueError("threshold is NaN")
        self.out_features, self.in_features = weight.shape
        weight = weight.to(torch.float16).contiguous()
        self.Wq, self.w_scale = int8_quant_weight(weight)
        self.W16 = weight if has_fp16_weights else None
        self.bias = None if bias is None else bias.to(torch.float16).contiguous()
        self.threshold = float(threshold)
        self.per_tensor_activation = bool(per_tensor_activation)
        self._workspace = None
        self._ws_rows = 0

    def _ws(self, M: int, device) -> torch.Tensor:
        if self._workspace is None or self._ws_rows < M:
            self._workspace = new_workspace(M, self.out_features, self.in_features, device)
            self._ws_rows = M
        return self._workspace

    def __call__(self, X: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        lead = X.shape[:-1]
        X2 = X.reshape(-1, self.in_features).contiguous()
        ws = self._ws(X2.shape[0], X2.device)
        if self.per_tensor_activation:
            Y = int8_linear_forward_ex(X2, self.Wq, self.w_scale, self.bias, self.threshold,
                                       W16=self.W16, per_tensor=True, Y=out, workspace=ws)
        elif self.W16 is not None:
            Y = int8_linear_forward_fp16w(X2, self.Wq, self.w_scale, self.W16, self.bias,
                                          self.threshold, Y=out, workspace=ws)
        else:
            Y = int8_linear_forward(X2, self.Wq, self.w_scale, self.bias, self.threshold, Y=out,
                                    workspace=ws)
        return Y.reshape(*lead, self.out_features)
