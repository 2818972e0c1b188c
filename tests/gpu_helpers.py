"""Shared helpers of the GPU parity tests (inputs from synth, references from the oracle)."""
import functools

import numpy as np
import torch

import synth

# Tolerance on Y: max |Y - Y_ref| <= 1e-2 * max |Y_ref| and ||Y - Y_ref||_2 <= 2e-3 ||Y_ref||_2.
# The integer stages (Wq, w_scale, outlier set, Xq, row scales, int32 accumulators, fp16
# outlier weights) are compared bit for bit.
MAX_ABS_REL = 1e-2
REL_L2 = 2e-3


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_y_close(Y: np.ndarray, Y_ref: np.ndarray, what: str = "Y") -> None:
    y = Y.astype(np.float64)
    r = Y_ref.astype(np.float64)
    assert np.isfinite(y).all(), f"{what}: non-finite values"
    scale = np.abs(r).max()
    err = np.abs(y - r).max()
    assert err <= MAX_ABS_REL * scale, f"{what}: max abs err {err} > {MAX_ABS_REL} * {scale}"
    l2 = np.linalg.norm(y - r) / max(np.linalg.norm(r), 1e-30)
    assert l2 <= REL_L2, f"{what}: relative L2 {l2} > {REL_L2}"


def f16_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, np.float16).view(np.uint16)


@functools.lru_cache(maxsize=4)
def workload_inputs(name: str, **changes):
    w = synth.WORKLOADS[name]
    if changes:
        w = synth.scaled(w, **changes)
    X, W, b, cols = synth.make_inputs(w)
    return w, X, W, b, cols


def sample_rows(M: int, n: int = 6, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    fixed = [0, M - 1, M // 2, min(M - 1, 127), min(M - 1, 128)]
    extra = rng.integers(0, M, size=max(0, n - len(fixed))).tolist()
    return np.unique(np.array(fixed + extra, np.int64))
