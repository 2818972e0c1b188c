"""The oracle against the naive float32 restatement, on layers that hypothesis searches for.

`naive_forward` (tests/test_oracle_bruteforce.py) restates the layer with numpy float32 array
arithmetic, independently of oracle/oracle.c.  Here hypothesis draws small layers from the
whole binary16 range instead of a fixed distribution: subnormal and large activations, exact
half-integer quotients (rows of (k + 1/2) 2^e with absmax 127 2^e), near half-integer quotients
for an arbitrary absmax a (the binary16 values nearest (k + 1/2) a / 127), zero rows, rows
whose only nonzero values are outliers, all-zero weight channels, and thresholds from 0 to
+inf.  Every integer stage must agree exactly and Y within one binary16 ulp ([P5] "PyTorch 2.9
支持 LLM.int8()" section "LLM.int8() 是怎么做到几乎无损的", items 1-3; [P2] "8位量化实战：
离群值处理与显存优化避坑指南" section 2.3).  The search is derandomized, so every run draws the
same examples.
"""
import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from tests.test_oracle_bruteforce import naive_forward


def half_bits(max_exp_field: int):
    """binary16 bit patterns with exponent field <= max_exp_field (0 gives zeros/subnormals)."""
    return st.builds(lambda s, e, m: (s << 15) | (e << 10) | m,
                     st.integers(0, 1), st.integers(0, max_exp_field), st.integers(0, 1023))


def as_half(bits, shape):
    return np.array(bits, dtype=np.uint16).reshape(shape).view(np.float16)


@st.composite
def layers(draw):
    M = draw(st.integers(1, 5))
    K = draw(st.sampled_from([8, 16]))
    N = draw(st.integers(1, 5))
    # |x| < 2^8 and |w| < 4 keep |Y| well inside binary16
    X = as_half(draw(st.lists(half_bits(22), min_size=M * K, max_size=M * K)), (M, K)).copy()
    W = as_half(draw(st.lists(half_bits(16), min_size=N * K, max_size=N * K)), (N, K)).copy()
    if draw(st.booleans()):  # a row of exact half-integer quotients
        i = draw(st.integers(0, M - 1))
        e = draw(st.integers(-20, 0))
        ks = draw(st.lists(st.integers(-126, 125), min_size=K, max_size=K))
        row = (np.array(ks, dtype=np.float64) + 0.5) * 2.0 ** e
        row[draw(st.integers(0, K - 1))] = 127 * 2.0 ** e
        X[i] = row.astype(np.float16)
    if draw(st.booleans()):  # near-half-integer quotients for an arbitrary binary16 absmax
        i = draw(st.integers(0, M - 1))
        a = float(as_half([draw(st.integers(0x1400, 0x5BFF))], (1,))[0])  # 2^-10 .. < 256
        # k = 63 or -64 puts x = +-a/2 exactly on the quotient 63.5: the case where x / s and
        # x * (127 / a) part ways
        ks = draw(st.lists(st.one_of(st.integers(-126, 125), st.sampled_from([63, -64])),
                           min_size=K, max_size=K))
        row = ((np.array(ks, dtype=np.float64) + 0.5) * (a / 127.0)).astype(np.float16)
        row[draw(st.integers(0, K - 1))] = np.float16(a)
        X[i] = row
    if draw(st.booleans()):  # outlier columns
        for j in draw(st.lists(st.integers(0, K - 1), max_size=3, unique=True)):
            X[draw(st.integers(0, M - 1)), j] = np.float16(draw(st.floats(8.0, 200.0)))
    if draw(st.booleans()):
        X[draw(st.integers(0, M - 1))] = 0
    if draw(st.booleans()):
        W[draw(st.integers(0, N - 1))] = 0
    b = None
    if draw(st.booleans()):
        b = as_half(draw(st.lists(half_bits(15), min_size=N, max_size=N)), (N,)).copy()
    t = draw(st.one_of(st.sampled_from([0.0, 1e-7, 0.5, 1.5, 6.0, 100.0, math.inf]),
                       st.floats(0.0, 300.0, width=32)))
    return X, W, b, float(t)


@settings(max_examples=400, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(layers())
def test_oracle_matches_naive_formulation_on_searched_layers(layer):
    X, W, b, t = layer
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
    assert np.isfinite(yr).all()
    ulp = np.spacing(np.abs(yr).astype(np.float16)).astype(np.float64)
    assert (np.abs(y - yr) <= ulp).all(), (X, W, b, t, Y, ref["Y"])
