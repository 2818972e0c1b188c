"""Seeded synthetic workloads for the LLM.int8() linear layer.

Shared by the tests, the oracle runs and bench.py; holds no arithmetic of the layer
itself (see synth.c for the generator's definition).  The workloads stand in for the
LLM activations the pages discuss: mostly N(0, sigma) features plus a few feature
columns scaled by a large factor, the emergent "outlier" dimensions of [P2]
"8位量化实战：离群值处理与显存优化避坑指南" section 2.2 and [P5] "PyTorch 2.9 支持
LLM.int8()" item 3 (0.01-0.1% of activations).
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

# stream ids (one independent random stream per tensor)
STREAM_X, STREAM_W, STREAM_BIAS, STREAM_COLS, STREAM_FACTORS, STREAM_SIGNS = 1, 2, 3, 4, 5, 6


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=gnu11", "-O2", "-fPIC", "-shared", "-fopenmp",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64, dbl, p = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.synth_u64.argtypes = [u64, u64]
            lib.synth_u64.restype = u64
            lib.synth_stream_key.argtypes = [u64, u64]
            lib.synth_stream_key.restype = u64
            lib.synth_uniform.argtypes = [u64, u64]
            lib.synth_uniform.restype = dbl
            lib.synth_normal.argtypes = [u64, u64]
            lib.synth_normal.restype = dbl
            lib.synth_normal_matrix_f16.argtypes = [u64, i64, i64, dbl, dbl, p, p]
            lib.synth_normal_matrix_f16.restype = None
            lib.synth_choose_distinct.argtypes = [u64, i64, i64, p, p]
            lib.synth_choose_distinct.restype = None
            _lib = lib
    return _lib


def stream_key(seed: int, stream: int) -> int:
    return int(_load().synth_stream_key(seed & (2**64 - 1), stream))


def uniform(key: int, index: int) -> float:
    return float(_load().synth_uniform(key, index))


def normal_f16(key: int, rows: int, cols: int, mean: float = 0.0, std: float = 1.0,
               col_factor: np.ndarray | None = None) -> np.ndarray:
    out = np.empty((rows, cols), np.float16)
    f = None
    if col_factor is not None:
        f = np.ascontiguousarray(col_factor, np.float64)
        assert f.shape == (cols,)
    _load().synth_normal_matrix_f16(key, rows, cols, mean, std,
                                    None if f is None else f.ctypes.data_as(ctypes.c_void_p),
                                    out.ctypes.data_as(ctypes.c_void_p))
    return out


def choose_distinct(key: int, n: int, count: int) -> np.ndarray:
    scratch = np.empty(n, np.int32)
    out = np.empty(count, np.int32)
    _load().synth_choose_distinct(key, n, count, scratch.ctypes.data_as(ctypes.c_void_p),
                                  out.ctypes.data_as(ctypes.c_void_p))
    return out


@dataclasses.dataclass(frozen=True)
class Workload:
    """One layer shape and its input distribution."""
    name: str
    M: int                      # tokens (rows of X)
    K: int                      # input features
    N: int                      # output channels
    x_std: float
    w_std: float
    bias_std: float | None      # None: no bias; 0.0: an all-zero bias vector
    threshold: float
    outlier_cols: tuple = ()    # fixed outlier columns, or () to draw n_outlier_cols at random
    n_outlier_cols: int = 0
    factor_lo: float = 20.0     # outlier columns are multiplied by U(factor_lo, factor_hi)
    factor_hi: float = 20.0
    random_sign: bool = False
    seed: int = 0

    @property
    def ops(self) -> float:
        """2*M*N*K, the operation count the throughput metric is quoted on."""
        return 2.0 * self.M * self.N * self.K

    @property
    def algorithmic_bytes(self) -> int:
        """Read X once, Wq once, the scales and bias once; write Y once."""
        b = self.M * self.K * 2 + self.N * self.K + self.N * 4 + self.M * self.N * 2
        if self.bias_std is not None:
            b += self.N * 2
        return b


def _fraction_cols(frac: float, K: int) -> int:
    return int(math.floor(frac * K + 0.5))


WORKLOADS = {
    "tiny": Workload("tiny", 16, 256, 256, 1.0, 0.02, 0.0, 6.0, outlier_cols=(7, 200),
                     factor_lo=20.0, factor_hi=20.0),
    "decode_q_proj": Workload("decode_q_proj", 8, 4096, 4096, 1.0, 0.02, None, 6.0,
                              n_outlier_cols=6, factor_lo=8.0, factor_hi=60.0, random_sign=True),
    "prefill_up_proj": Workload("prefill_up_proj", 2048, 4096, 11008, 1.0, 0.02, 0.01, 6.0,
                                n_outlier_cols=_fraction_cols(0.0015, 4096), factor_lo=8.0,
                                factor_hi=60.0),
    "down_proj_13b": Workload("down_proj_13b", 4096, 13824, 5120, 0.5, 0.015, None, 6.0,
                              n_outlier_cols=12, factor_lo=10.0, factor_hi=80.0),
}
for _frac in (0.0, 0.001, 0.01):
    for _t in (0.0, 6.0, math.inf):
        _name = f"ffn_175b_f{_frac:g}_t{_t:g}"
        WORKLOADS[_name] = Workload(_name, 2048, 12288, 49152, 1.0, 0.01, None, _t,
                                    n_outlier_cols=_fraction_cols(_frac, 12288), factor_lo=8.0,
                                    factor_hi=60.0)


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (e.g. smaller M for a test)."""
    return dataclasses.replace(w, **changes)


def make_inputs(w: Workload, seed: int | None = None):
    """X (float16 [M,K]), W (float16 [N,K]), bias (float16 [N] or None), outlier columns."""
    seed = w.seed if seed is None else seed
    if w.outlier_cols:
        cols = np.array(w.outlier_cols, np.int32)
    else:
        cols = choose_distinct(stream_key(seed, STREAM_COLS), w.K, w.n_outlier_cols)
    factor = np.ones(w.K, np.float64)
    fkey = stream_key(seed, STREAM_FACTORS)
    skey = stream_key(seed, STREAM_SIGNS)
    for r, j in enumerate(cols):
        f = w.factor_lo + (w.factor_hi - w.factor_lo) * uniform(fkey, r)
        if w.random_sign and uniform(skey, r) < 0.5:
            f = -f
        factor[j] = f
    X = normal_f16(stream_key(seed, STREAM_X), w.M, w.K, 0.0, w.x_std, factor)
    W = normal_f16(stream_key(seed, STREAM_W), w.N, w.K, 0.0, w.w_std)
    bias = None
    if w.bias_std is not None:
        bias = normal_f16(stream_key(seed, STREAM_BIAS), 1, w.N, 0.0, w.bias_std).reshape(w.N)
    return X, W, bias, cols
