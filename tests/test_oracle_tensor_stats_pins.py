"""Pins of the oracle's per-tensor activation scale ([P5] "PyTorch 2.9 支持 LLM.int8()" item 2,
whose snippet takes one absmax over the whole tensor) and of its activation statistics ([P2]
"8位量化实战：离群值处理与显存优化避坑指南" section 5.1: max, 0.99 quantile and their ratio).

- one row: the per-tensor layer is the per-row layer, bit for bit;
- rows sharing one regular absmax: both give the same codes and Y;
- the tensor scale is the largest of the row scales (x / 127 is monotone), in every row;
- a naive numpy float32 restatement on many 4 x 8 layers agrees exactly on the codes and
  scales and within one binary16 ulp on Y;
- the decomposition's error bound holds with the tensor scale;
- statistics: the closed form of 0..99 (q99 = 98.01), numpy's linear quantile, the column
  absmax and max exactly, one element.
"""
import math

import numpy as np
import pytest

import oracle


def layer(seed, M=6, K=40, N=5, n_out=2, factor=30.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K)) * rng.uniform(0.2, 3.0, size=(M, 1))
    cols = rng.choice(K, size=n_out, replace=False)
    X[:, cols] *= factor
    W = rng.standard_normal((N, K)) * 0.05
    b = (rng.standard_normal(N) * 0.1).astype(np.float16)
    return X.astype(np.float16), W.astype(np.float16), b


@pytest.mark.parametrize("seed", range(3))
def test_one_row_per_tensor_is_per_row(seed):
    X, W, b = layer(seed, M=1)
    Wq, sw = oracle.quant_weight(W)
    rows = np.arange(1)
    Y_t, A_t = oracle.linear_forward_rows_ex(X, Wq, sw, b, 6.0, rows, per_tensor=True)
    Y_r, A_r = oracle.linear_forward_rows(X, Wq, sw, b, 6.0, rows)
    np.testing.assert_array_equal(A_t, A_r)
    np.testing.assert_array_equal(Y_t.view(np.uint16), Y_r.view(np.uint16))


def test_rows_sharing_one_absmax_give_the_per_row_layer():
    X, W, b = layer(7, M=5, n_out=0)
    X = X.astype(np.float64)
    X /= np.abs(X).max(axis=1, keepdims=True)   # every row's absmax is 1
    X = (X * 2.5).astype(np.float16)
    Wq, sw = oracle.quant_weight(W)
    mask, _ = oracle.outlier_columns(X, 6.0)
    Xq_t, s_t = oracle.quantize_tensor(X, mask)
    Xq_r, s_r = oracle.quantize_rows(X, mask)
    np.testing.assert_array_equal(Xq_t, Xq_r)
    np.testing.assert_array_equal(s_t.view(np.uint32), s_r.view(np.uint32))
    np.testing.assert_array_equal(oracle.linear_forward_tensor(X, Wq, sw, b, 6.0).view(np.uint16),
                                  oracle.linear_forward(X, Wq, sw, b, 6.0).view(np.uint16))


@pytest.mark.parametrize("seed", range(4))
def test_tensor_scale_is_the_largest_row_scale(seed):
    X, _, _ = layer(30 + seed)
    mask, _ = oracle.outlier_columns(X, 6.0)
    _, s_r = oracle.quantize_rows(X, mask)
    _, s_t = oracle.quantize_tensor(X, mask)
    assert np.all(s_t == s_r.max())


def naive_tensor_forward(X, W, b, t):
    x = X.astype(np.float32)
    w = W.astype(np.float32)
    aw = np.abs(w).max(axis=1)
    sw = aw / np.float32(127.0)
    safe_sw = np.where(sw == 0, np.float32(1.0), sw)
    Wq = np.where(aw[:, None] == 0, 0, np.clip(np.rint(w / safe_sw[:, None]), -127, 127)).astype(np.int8)
    tt = np.float32(max(t, 0.0)) if not math.isinf(t) else np.float32(np.inf)
    outl = (np.abs(x) > tt).any(axis=0)
    ax = np.float32(np.where(outl[None, :], np.float32(0.0), np.abs(x)).max())
    s = ax / np.float32(127.0)
    Xq = np.clip(np.rint(x / (s if s != 0 else np.float32(1.0))), -127, 127)
    Xq = np.where(outl[None, :] | (ax == 0), 0, Xq).astype(np.int8)
    A = Xq.astype(np.int64) @ Wq.astype(np.int64).T
    W_hat = (Wq.astype(np.float32) * sw[:, None]).astype(np.float16)
    P = X[:, outl].astype(np.float64) @ W_hat[:, outl].astype(np.float64).T
    Y = A.astype(np.float64) * np.float64(s) * sw.astype(np.float64)[None, :] + P
    if b is not None:
        Y = Y + b.astype(np.float64)[None, :]
    return Xq, s, A, Y.astype(np.float16)


@pytest.mark.parametrize("seed", range(6))
def test_naive_float32_restatement_on_4x8_layers(seed):
    rng = np.random.default_rng(500 + seed)
    for _ in range(40):
        M, K, N = 4, 8, 5
        X = rng.standard_normal((M, K)) * rng.uniform(0.1, 3.0, size=(M, 1))
        cols = rng.choice(K, size=rng.integers(0, 3), replace=False)
        X[:, cols] *= rng.uniform(8, 60)
        # exact half-integer quotients in one row: scale 2^-3 set by a 127 * 2^-3 entry
        i = rng.integers(0, M)
        reg = [j for j in range(K) if j not in set(cols.tolist())]
        if reg:
            X[i, reg] = (rng.integers(-126, 126, size=len(reg)) + 0.5) * 0.125
            X[i, reg[0]] = 127 * 0.125
            X[np.ix_(np.flatnonzero(np.arange(M) != i), reg)] *= 0.5
        X = X.astype(np.float16)
        W = (rng.standard_normal((N, K)) * 0.05).astype(np.float16)
        b = (rng.standard_normal(N) * 0.1).astype(np.float16) if rng.random() < 0.7 else None
        t = float(rng.choice([6.0, 1.5, 0.0, math.inf]))
        Xq_n, s_n, A_n, Y_n = naive_tensor_forward(X, W, b, t)
        Wq, sw = oracle.quant_weight(W)
        mask, _ = oracle.outlier_columns(X, t)
        Xq, s = oracle.quantize_tensor(X, mask)
        np.testing.assert_array_equal(Xq, Xq_n)
        assert np.all(s.view(np.uint32) == np.float32(s_n).view(np.uint32))
        Y, A = oracle.linear_forward_rows_ex(X, Wq, sw, b, t, np.arange(M), per_tensor=True)
        np.testing.assert_array_equal(A.astype(np.int64), A_n)
        y, yn = Y.astype(np.float64), Y_n.astype(np.float64)
        assert (np.abs(y - yn) <= np.spacing(np.abs(Y_n)).astype(np.float64)).all()


def test_error_bound_with_the_tensor_scale():
    X, W, b = layer(77, M=12, K=96, N=9, n_out=3)
    Wq, sw = oracle.quant_weight(W)
    mask, cols = oracle.outlier_columns(X, 6.0)
    _, s = oracle.quantize_tensor(X, mask)
    Y = oracle.linear_forward_tensor(X, Wq, sw, b, 6.0).astype(np.float64)
    x, w = X.astype(np.float64), W.astype(np.float64)
    exact = x @ w.T + b.astype(np.float64)
    r = np.ones(X.shape[1], bool)
    r[cols] = False
    sd, swd = float(s[0]), sw.astype(np.float64)[None, :]
    W_hat = oracle.outlier_weights(Wq, sw, cols).astype(np.float64)
    bound = (np.abs(x[:, r]).sum(1)[:, None] * swd / 2 + np.abs(w[:, r]).sum(1)[None, :] * sd / 2
             + r.sum() * sd * swd / 4) * (1 + 1e-5)
    bound += np.abs(x[:, cols]) @ np.abs(w[:, cols] - W_hat).T
    bound += np.spacing(np.abs(Y).astype(np.float16)).astype(np.float64)
    assert (np.abs(Y - exact) <= bound).all()


def test_stats_closed_form_of_0_to_99():
    X = np.arange(100, dtype=np.float16).reshape(4, 25)
    mx, q99, ratio, col = oracle.activation_stats(X)
    assert mx == 99.0
    assert abs(q99 - 98.01) < 1e-12
    assert ratio == 99.0 / (q99 + 1e-6)
    np.testing.assert_array_equal(col, np.arange(75, 100, dtype=np.float32))


@pytest.mark.parametrize("seed", range(4))
def test_stats_against_numpy_quantile(seed):
    rng = np.random.default_rng(seed)
    M, K = rng.integers(1, 40), rng.integers(1, 300)
    X = (rng.standard_normal((M, K)) * rng.uniform(0.1, 50)).astype(np.float16)
    mx, q99, ratio, col = oracle.activation_stats(X)
    a = np.abs(X.astype(np.float64))
    assert mx == a.max()
    assert abs(q99 - np.quantile(a, 0.99)) <= 1e-12 * max(1.0, a.max())
    np.testing.assert_array_equal(col, a.max(axis=0).astype(np.float32))
    assert ratio == mx / (q99 + 1e-6)


def test_stats_of_one_element():
    mx, q99, ratio, col = oracle.activation_stats(np.array([[-3.5]], np.float16))
    assert (mx, q99) == (3.5, 3.5) and col[0] == 3.5
