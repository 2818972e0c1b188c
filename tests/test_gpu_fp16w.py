"""GPU parity of the layer that keeps its fp16 weights (int8_linear_forward_fp16w) against the
oracle's linear_forward_w16, on every route the forward takes: the one-launch decode kernel
(M <= 8), the few-token GEMV (M <= 16), the cluster kernel for long rows, and the tiled
tensor-core GEMM.

Two properties besides the tolerance on Y:
- kept weights equal to the rebuilt fp16(Wq * w_scale) give the default layer's Y bit for bit
  (the same kernels read the same fp16 values);
- on layers with very large outlier columns, the result is far closer to the kept-weight
  reference than to the default layer's, so the kernels did read W16.
"""
import math

import numpy as np
import pytest
import torch

import int8_mixed_precision_absmax_b200 as i8
import oracle
from tests.gpu_helpers import assert_y_close, f16_bits, to_dev, to_np

pytestmark = pytest.mark.gpu

SHAPES = [
    (8, 4096, 4096, 6, 6.0),     # decode kernel
    (5, 4096, 256, 40, 6.0),     # decode kernel, many outlier columns
    (8, 1024, 1024, 0, 0.0),     # decode kernel, every column an outlier
    (12, 2048, 640, 5, 6.0),     # few-token GEMV
    (16, 256, 128, 3, 0.0),      # few-token GEMV, every column an outlier
    (5, 20000, 200, 4, 6.0),     # long rows (cluster kernel)
    (16, 16384, 300, 4, 6.0),    # long rows (cluster kernel)
    (200, 1040, 600, 5, 6.0),    # tiled GEMM
    (300, 512, 384, 0, 0.0),     # tiled GEMM, every column an outlier
    (64, 256, 256, 2, math.inf),  # no outlier term at all
]


def case(M, K, N, n_out, seed, factor=20.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    cols = rng.choice(K, size=n_out, replace=False) if n_out else []
    X[:, cols] *= factor
    W = rng.standard_normal((N, K)) * 0.02
    b = (rng.standard_normal(N) * 0.01).astype(np.float16)
    return X.astype(np.float16), W.astype(np.float16), b


def gpu_forward(X, W16, b, t, fp16w=True):
    Xd = to_dev(X)
    Wq, sw = i8.int8_quant_weight(to_dev(W16))
    ws = i8.new_workspace(X.shape[0], W16.shape[0], X.shape[1], Xd.device)
    if fp16w:
        Y = i8.int8_linear_forward_fp16w(Xd, Wq, sw, to_dev(W16), to_dev(b), t, workspace=ws)
    else:
        Y = i8.int8_linear_forward(Xd, Wq, sw, to_dev(b), t, workspace=ws)
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0
    torch.cuda.synchronize()
    return to_np(Y)


@pytest.mark.parametrize("M,K,N,n_out,t", SHAPES)
def test_fp16w_forward_matches_oracle(M, K, N, n_out, t):
    X, W, b = case(M, K, N, n_out, seed=M + 5 * K + 11 * N)
    Wq, sw = oracle.quant_weight(W)
    Y_ref = oracle.linear_forward_w16(X, Wq, sw, W, b, t)
    assert_y_close(gpu_forward(X, W, b, t), Y_ref, f"fp16w {M}x{K}x{N} t={t}")


@pytest.mark.parametrize("M,K,N,n_out,t", [s for s in SHAPES if s[3] or s[4] == 0.0])
def test_rebuilt_weights_give_the_default_layer_bit_for_bit(M, K, N, n_out, t):
    X, W, b = case(M, K, N, n_out, seed=7 * M + K + N)
    Wq, sw = oracle.quant_weight(W)
    W_hat = (Wq.astype(np.float32) * sw[:, None]).astype(np.float16)
    Y_w = gpu_forward(X, W_hat, b, t)
    Y_d = gpu_forward(X, W_hat, b, t, fp16w=False)
    np.testing.assert_array_equal(f16_bits(Y_w), f16_bits(Y_d))


@pytest.mark.parametrize("M,K,N", [(8, 4096, 1024), (12, 2048, 640), (16, 16384, 300),
                                   (256, 1024, 512)])
def test_kernels_read_the_kept_weights(M, K, N):
    X, W, b = case(M, K, N, 3, seed=M * K + N, factor=2000.0)
    Wq, sw = oracle.quant_weight(W)
    Y_w16 = oracle.linear_forward_w16(X, Wq, sw, W, b, 6.0).astype(np.float64)
    Y_def = oracle.linear_forward(X, Wq, sw, b, 6.0).astype(np.float64)
    Y = gpu_forward(X, W, b, 6.0).astype(np.float64)
    gap = np.abs(Y_def - Y_w16).max()
    assert gap > 0
    assert np.abs(Y - Y_w16).max() < gap / 4
