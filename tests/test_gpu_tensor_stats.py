"""GPU parity of the per-tensor activation scale (int8_linear_forward_ex with
PER_TENSOR_SCALE) and of the activation statistics (int8_activation_stats) against the
oracle, on every route of the forward (decode kernel, few-token GEMV, long-row cluster
kernel, tiled GEMM)."""
import math

import numpy as np
import pytest
import torch

import int8_mixed_precision_absmax_b200 as i8
import oracle
import synth
from tests.gpu_helpers import assert_y_close, f16_bits, to_dev, to_np

pytestmark = pytest.mark.gpu

SHAPES = [
    (8, 4096, 4096, 6, 6.0),     # decode kernel
    (5, 1024, 200, 3, 6.0),      # decode kernel, ragged channels
    (12, 2048, 640, 5, 6.0),     # few-token GEMV
    (16, 16384, 300, 4, 6.0),    # long rows (cluster kernel)
    (200, 1040, 600, 5, 6.0),    # tiled GEMM
    (300, 512, 384, 0, 0.0),     # tiled, every column an outlier
    (64, 4096, 256, 2, math.inf),  # tiled, no outlier term
]


def case(M, K, N, n_out, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K)) * rng.uniform(0.1, 4.0, size=(M, 1))  # rows of unequal range
    cols = rng.choice(K, size=n_out, replace=False) if n_out else []
    X[:, cols] *= 25.0
    W = rng.standard_normal((N, K)) * 0.02
    b = (rng.standard_normal(N) * 0.01).astype(np.float16)
    return X.astype(np.float16), W.astype(np.float16), b


def gpu_ex(X, W, b, t, per_tensor, W16=None):
    Xd = to_dev(X)
    Wq, sw = i8.int8_quant_weight(to_dev(W))
    M, N = X.shape[0], W.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    ws = i8.new_workspace(M, N, X.shape[1], Xd.device)
    Y = i8.int8_linear_forward_ex(Xd, Wq, sw, to_dev(b), t, W16=None if W16 is None else to_dev(W16),
                                  per_tensor=per_tensor, acc=acc, workspace=ws)
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0
    torch.cuda.synchronize()
    return to_np(Y), to_np(acc), to_np(Wq), to_np(sw)


@pytest.mark.parametrize("M,K,N,n_out,t", SHAPES)
@pytest.mark.parametrize("kept", [False, True])
def test_per_tensor_forward_matches_oracle(M, K, N, n_out, t, kept):
    X, W, b = case(M, K, N, n_out, seed=M + 3 * K + N + kept)
    Y, acc, Wq, sw = gpu_ex(X, W, b, t, True, W16=W if kept else None)
    Y_ref, A_ref = oracle.linear_forward_rows_ex(X, Wq, sw, b, t, np.arange(M),
                                                 W16=W if kept else None, per_tensor=True)
    np.testing.assert_array_equal(acc, A_ref)
    assert_y_close(Y, Y_ref, f"per-tensor {M}x{K}x{N} t={t} kept={kept}")


@pytest.mark.parametrize("M,K,N,n_out,t", [SHAPES[0], SHAPES[2], SHAPES[4]])
def test_per_row_default_unchanged_by_the_extended_entry(M, K, N, n_out, t):
    X, W, b = case(M, K, N, n_out, seed=11 * M + K)
    Y_ex, acc_ex, Wq, sw = gpu_ex(X, W, b, t, False)
    Y_ref, A_ref = oracle.linear_forward_rows(X, Wq, sw, b, t, np.arange(M))
    np.testing.assert_array_equal(acc_ex, A_ref)
    Y = to_np(i8.int8_linear_forward(to_dev(X), to_dev(Wq), to_dev(sw), to_dev(b), t))
    np.testing.assert_array_equal(f16_bits(Y_ex), f16_bits(Y))


@pytest.mark.parametrize("M,K", [(1, 256), (8, 4096), (13, 2048), (300, 1040), (2048, 4096)])
def test_activation_stats_match_oracle(M, K):
    rng = np.random.default_rng(M * 7 + K)
    X = rng.standard_normal((M, K)) * 0.8
    X[:, rng.choice(K, size=3, replace=False)] *= 40.0
    X = X.astype(np.float16)
    out, col = i8.int8_activation_stats(to_dev(X))
    torch.cuda.synchronize()
    mx, q99, ratio, col_ref = oracle.activation_stats(X)
    o = to_np(out)
    assert o[0] == mx and o[1] == q99 and o[2] == ratio, (o, mx, q99, ratio)
    np.testing.assert_array_equal(to_np(col), col_ref)


def test_activation_stats_on_the_prefill_workload():
    w = synth.WORKLOADS["prefill_up_proj"]
    X, _, _, _ = synth.make_inputs(w)
    out, col = i8.int8_activation_stats(to_dev(X))
    torch.cuda.synchronize()
    mx, q99, ratio, col_ref = oracle.activation_stats(X)
    np.testing.assert_array_equal(to_np(out), np.array([mx, q99, ratio]))
    np.testing.assert_array_equal(to_np(col), col_ref)
    # the outlier columns of the layer are the columns whose absmax exceeds the threshold
    _, cols = oracle.outlier_columns(X, w.threshold)
    np.testing.assert_array_equal(np.flatnonzero(to_np(col) > w.threshold), cols)
