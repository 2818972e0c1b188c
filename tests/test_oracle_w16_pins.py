"""Pins of the oracle's kept-fp16-weights variant ([P5] "如何在 PyTorch 2.9 中启用 LLM.int8 推理",
has_fp16_weights=True): the outlier columns use the layer's own fp16 weights.

- threshold 0 (every column an outlier): the layer is the fp16 product X . W^T + b, summed
  exactly enough in double: it equals numpy's float64 product rounded to fp16 within one ulp;
- kept weights equal to the rebuilt fp16(Wq * w_scale): the variant is the default layer, bit
  for bit; threshold +inf (no outliers): likewise;
- with the original weights the outlier term carries no weight-quantization error, so the
  error against the exact product obeys a bound with no outlier-weight term: a variant that
  ignored the kept weights breaks it on a layer with a large outlier column.
"""
import math

import numpy as np
import pytest

import oracle


def layer(seed, M=5, K=48, N=7, n_out=2, factor=40.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    cols = rng.choice(K, size=n_out, replace=False)
    X[:, cols] *= factor
    W = rng.standard_normal((N, K)) * 0.05
    b = (rng.standard_normal(N) * 0.1).astype(np.float16)
    return X.astype(np.float16), W.astype(np.float16), b, cols


@pytest.mark.parametrize("seed", range(3))
def test_threshold_zero_is_the_fp16_product_of_the_kept_weights(seed):
    X, W, b, _ = layer(seed)
    Wq, sw = oracle.quant_weight(W)
    Y = oracle.linear_forward_w16(X, Wq, sw, W, b, 0.0).astype(np.float64)
    ref = (X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)).astype(np.float16)
    ulp = np.spacing(np.abs(ref)).astype(np.float64)
    assert (np.abs(Y - ref.astype(np.float64)) <= ulp).all()


@pytest.mark.parametrize("t", [6.0, 0.0, math.inf])
def test_kept_weights_equal_to_the_rebuilt_ones_give_the_default_layer(t):
    X, W, b, _ = layer(11)
    Wq, sw = oracle.quant_weight(W)
    W_rebuilt = (Wq.astype(np.float32) * sw[:, None]).astype(np.float16)
    Y_def = oracle.linear_forward(X, Wq, sw, b, t)
    Y_w16 = oracle.linear_forward_w16(X, Wq, sw, W_rebuilt, b, t)
    np.testing.assert_array_equal(Y_w16.view(np.uint16), Y_def.view(np.uint16))


def test_threshold_inf_ignores_the_kept_weights():
    X, W, b, _ = layer(12)
    Wq, sw = oracle.quant_weight(W)
    np.testing.assert_array_equal(oracle.linear_forward_w16(X, Wq, sw, W, b, math.inf).view(np.uint16),
                                  oracle.linear_forward(X, Wq, sw, b, math.inf).view(np.uint16))


@pytest.mark.parametrize("seed", range(3))
def test_error_bound_without_an_outlier_weight_term(seed):
    X, W, b, cols = layer(20 + seed, factor=1000.0)
    Wq, sw = oracle.quant_weight(W)
    mask, found = oracle.outlier_columns(X, 6.0)
    np.testing.assert_array_equal(np.sort(cols), found)
    _, sx = oracle.quantize_rows(X, mask)
    Y = oracle.linear_forward_w16(X, Wq, sw, W, b, 6.0).astype(np.float64)
    x, w = X.astype(np.float64), W.astype(np.float64)
    exact = x @ w.T + b.astype(np.float64)
    r = np.ones(X.shape[1], bool)
    r[found] = False
    sxd, swd = sx.astype(np.float64)[:, None], sw.astype(np.float64)[None, :]
    bound = (np.abs(x[:, r]).sum(1)[:, None] * swd / 2 + np.abs(w[:, r]).sum(1)[None, :] * sxd / 2
             + r.sum() * sxd * swd / 4) * (1 + 1e-5)
    bound += np.spacing(np.abs(Y).astype(np.float16)).astype(np.float64)
    assert (np.abs(Y - exact) <= bound).all()
    # the rebuilt weights of the same layer exceed that bound: the kept weights are what the
    # variant used
    Y_def = oracle.linear_forward(X, Wq, sw, b, 6.0).astype(np.float64)
    assert (np.abs(Y_def - exact) > bound).any()
