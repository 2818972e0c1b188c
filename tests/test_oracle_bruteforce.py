"""The oracle against a second, deliberately naive formulation, and against the exact product
on the benchmark workloads.

`naive_forward` restates the layer with numpy float32 arithmetic and whole-array operations
(IEEE float32 divisions, np.rint for round-half-to-even, np.clip), written independently of
oracle/oracle.c.  On many random 4 x 8 layers with planted outlier columns and activations
placed exactly on half-integer quotients, every integer stage must agree exactly and Y to
within one binary16 ulp.  The error bound of the decomposition (each regular product term off
by at most half a quantization step on each side, each outlier term by the fp16 rounding of
the rebuilt weight) is then checked element by element on whole benchmark workloads.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def naive_forward(X, W, b, t):
    x = X.astype(np.float32)
    w = W.astype(np.float32)
    aw = np.abs(w).max(axis=1)
    sw = aw / np.float32(127.0)
    safe_sw = np.where(sw == 0, np.float32(1.0), sw)
    Wq = np.where(aw[:, None] == 0, 0, np.clip(np.rint(w / safe_sw[:, None]), -127, 127))
    Wq = Wq.astype(np.int8)
    tt = np.float32(max(t, 0.0)) if not math.isinf(t) else np.float32(np.inf)
    outl = (np.abs(x) > tt).any(axis=0)
    xr = np.where(outl[None, :], np.float32(0.0), np.abs(x))
    ax = xr.max(axis=1)
    sx = ax / np.float32(127.0)
    safe_sx = np.where(sx == 0, np.float32(1.0), sx)
    Xq = np.clip(np.rint(x / safe_sx[:, None]), -127, 127)
    Xq = np.where(outl[None, :] | (ax[:, None] == 0), 0, Xq).astype(np.int8)
    A = Xq.astype(np.int64) @ Wq.astype(np.int64).T
    W_hat = (Wq.astype(np.float32) * sw[:, None]).astype(np.float16)
    P = X[:, outl].astype(np.float64) @ W_hat[:, outl].astype(np.float64).T
    Y = A.astype(np.float64) * sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :] + P
    if b is not None:
        Y = Y + b.astype(np.float64)[None, :]
    return dict(Wq=Wq, sw=sw, outl=outl, Xq=Xq, sx=sx, A=A, Y=Y.astype(np.float16))


def random_tiny_layer(rng):
    M, K, N = 4, 8, 5
    X = rng.standard_normal((M, K)) * rng.choice([0.5, 1.0, 2.0])
    n_out = rng.integers(0, 3)
    cols = rng.choice(K, size=n_out, replace=False)
    X[:, cols] *= rng.uniform(8, 60, size=n_out) * rng.choice([-1, 1], size=n_out)
    # one row whose quotients are exact half-integers: absmax 127 * 2^-3, entries (k + 1/2) 2^-3
    i = rng.integers(0, M)
    s = 2.0 ** -3
    regular = [j for j in range(K) if j not in set(cols.tolist())]
    if regular:
        X[i, regular] = (rng.integers(-126, 126, size=len(regular)) + 0.5) * s
        X[i, regular[0]] = 127 * s
    W = rng.standard_normal((N, K)) * 0.05
    if rng.random() < 0.2:
        W[rng.integers(0, N)] = 0.0
    b = (rng.standard_normal(N) * 0.1).astype(np.float16) if rng.random() < 0.7 else None
    t = float(rng.choice([6.0, 1.5, 0.0, math.inf]))
    return X.astype(np.float16), W.astype(np.float16), b, t


@pytest.mark.parametrize("seed", range(8))
def test_oracle_matches_naive_float32_formulation_on_4x8_layers(seed):
    rng = np.random.default_rng(1000 + seed)
    for _ in range(40):
        X, W, b, t = random_tiny_layer(rng)
        ref = naive_forward(X, W, b, t)
        Wq, sw = oracle.quant_weight(W)
        np.testing.assert_array_equal(Wq, ref["Wq"])
        np.testing.assert_array_equal(sw.view(np.uint32), ref["sw"].view(np.uint32))
        mask, cols = oracle.outlier_columns(X, t)
        np.testing.assert_array_equal(np.flatnonzero(ref["outl"]), cols)
        Xq, sx = oracle.quantize_rows(X, mask)
        np.testing.assert_array_equal(Xq, ref["Xq"])
        np.testing.assert_array_equal(sx.view(np.uint32), ref["sx"].view(np.uint32))
        np.testing.assert_array_equal(oracle.gemm_i32(Xq, Wq).astype(np.int64), ref["A"])
        Y = oracle.linear_forward(X, Wq, sw, b, t)
        y, yr = Y.astype(np.float64), ref["Y"].astype(np.float64)
        ulp = np.spacing(np.abs(yr).astype(np.float16)).astype(np.float64)
        assert (np.abs(y - yr) <= ulp).all(), (X, W, b, t, Y, ref["Y"])


def error_bound_holds(X, W, b, t, rows=None):
    Wq, sw = oracle.quant_weight(W)
    mask, cols = oracle.outlier_columns(X, t)
    Xq, sx = oracle.quantize_rows(X, mask)
    if rows is None:
        rows = np.arange(X.shape[0])
    Y, _ = oracle.linear_forward_rows(X, Wq, sw, b, t, rows)
    Y = Y.astype(np.float64)
    x = X[rows].astype(np.float64)
    w = W.astype(np.float64)
    exact = x @ w.T + (0.0 if b is None else b.astype(np.float64)[None, :])
    K = X.shape[1]
    out = np.zeros(K, bool)
    out[cols] = True
    sxd = sx[rows].astype(np.float64)[:, None]
    swd = sw.astype(np.float64)[None, :]
    W_hat = (Wq.astype(np.float32) * sw[:, None]).astype(np.float16).astype(np.float64)
    ulp_hat = np.spacing(np.abs(W_hat).astype(np.float16)).astype(np.float64)
    ax_r = np.abs(x[:, ~out]).sum(axis=1)[:, None]
    aw_r = np.abs(w[:, ~out]).sum(axis=1)[None, :]
    n_r = float((~out).sum())
    bound = (ax_r * swd / 2 + aw_r * sxd / 2 + n_r * sxd * swd / 4) * (1 + 1e-5)
    if out.any():
        bound += np.abs(x[:, out]) @ (swd / 2 + ulp_hat[:, out].T)
    bound += np.spacing(np.abs(Y).astype(np.float16)).astype(np.float64)
    return bool((np.abs(Y - exact) <= bound).all())


@pytest.mark.parametrize("name", ["tiny", "decode_q_proj"])
def test_error_bound_on_whole_workloads(name):
    w = synth.WORKLOADS[name]
    X, W, b, _ = synth.make_inputs(w)
    assert error_bound_holds(X, W, b, w.threshold)


def test_error_bound_on_prefill_rows():
    w = synth.WORKLOADS["prefill_up_proj"]
    X, W, b, _ = synth.make_inputs(w)
    assert error_bound_holds(X, W, b, w.threshold, rows=np.array([0, 1, 1023, 2047]))
