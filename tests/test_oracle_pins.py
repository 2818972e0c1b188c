"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against something it cannot have produced: a hand-worked
example (tests/golden/, with its citation), a closed form, an invariant of the
definitions, a special case that reduces to a library routine (numpy), or the exact
product within the method's error bound.  Together they are chosen so that a plausible
slip in the oracle (rounding mode, scale formula, clamp range, strict vs. non-strict
threshold, row maximum taken over the wrong columns, transposed operand, dropped bias or
outlier term, int32 overflow) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            rows = [r.split() for r in val.split(";")]
            out[key.strip()] = rows
    return out


def arr(rows, dtype):
    a = np.array([[float(v) for v in r] for r in rows], dtype=np.float64)
    return a.astype(dtype)


def f16_bits(a):
    return np.ascontiguousarray(a, np.float16).view(np.uint16)


def fl32_div(a, b):
    """Correctly rounded float32 quotient, computed without any float32 division:
    a float64 quotient of float32 operands rounded once more to float32 is correctly
    rounded (53 >= 2*24 + 2)."""
    return np.float32(float(a) / float(b))


# --------------------------------------------------------------------------- binary16

def test_half_decode_exhaustive_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_half_encode_matches_numpy_rounding():
    rng = np.random.default_rng(1)
    finite = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    nxt = np.arange(1, 0x7C01, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (finite + nxt) / 2                       # exact ties between neighbours
    near = np.concatenate([np.nextafter(mids, 0), np.nextafter(mids, np.inf)])
    randoms = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000),
        np.array([65504.0, 65519.99, 65520.0, 65536.0, 1e9, 2.0**-24, 2.0**-25,
                  3 * 2.0**-26, 2.0**-26, 2.0**-14, 2.0**-14 - 2.0**-25, 0.0, -0.0]),
    ])
    xs = np.concatenate([finite[::7], mids[::3], near[::5], randoms])
    xs = np.concatenate([xs, -xs])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.half_from_double(float(x)) for x in xs], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(xs[i], hex(got[i]), hex(ref[i])) for i in bad[:5]]


# --------------------------------------------------------------------------- hand-worked

def test_hand_example_round_half_even():
    g = load_golden("hand_rne_row.txt")
    X = arr(g["X"], np.float16)
    mask, cols = oracle.outlier_columns(X, float(g["threshold"][0][0]))
    assert cols.size == 0
    Xq, sx = oracle.quantize_rows(X, mask)
    assert sx[0] == np.float32(g["row_scale"][0][0])
    np.testing.assert_array_equal(Xq, arr(g["Xq"], np.int8))


def test_hand_example_divides_by_the_scale():
    g = load_golden("hand_scale_quotient.txt")
    X = arr(g["X"], np.float16)
    mask, cols = oracle.outlier_columns(X, float(g["threshold"][0][0]))
    Xq, _ = oracle.quantize_rows(X, mask)
    np.testing.assert_array_equal(Xq, arr(g["Xq"], np.int8))


def test_hand_example_decomposition_every_stage():
    g = load_golden("hand_decomposition.txt")
    X = arr(g["X"], np.float16)
    W = arr(g["W"], np.float16)
    t = float(g["threshold"][0][0])
    Wq, sw = oracle.quant_weight(W)
    np.testing.assert_array_equal(Wq, arr(g["Wq"], np.int8))
    np.testing.assert_array_equal(sw, arr(g["w_scale"], np.float32).ravel())
    mask, cols = oracle.outlier_columns(X, t)
    np.testing.assert_array_equal(cols, arr(g["outlier_cols"], np.int32).ravel())
    Xq, sx = oracle.quantize_rows(X, mask)
    np.testing.assert_array_equal(Xq, arr(g["Xq"], np.int8))
    np.testing.assert_array_equal(sx, arr(g["row_scale"], np.float32).ravel())
    A = oracle.gemm_i32(Xq, Wq)
    np.testing.assert_array_equal(A, arr(g["A"], np.int32))
    W_hat = oracle.outlier_weights(Wq, sw, cols)
    np.testing.assert_array_equal(f16_bits(W_hat), f16_bits(arr(g["W_hat"], np.float16)))
    Y = oracle.linear_forward(X, Wq, sw, None, t)
    np.testing.assert_array_equal(f16_bits(Y), f16_bits(arr(g["Y"], np.float16)))
    Y_rows, A_rows = oracle.linear_forward_rows(X, Wq, sw, None, t, [1])
    np.testing.assert_array_equal(f16_bits(Y_rows), f16_bits(Y[1:2]))
    np.testing.assert_array_equal(A_rows, A[1:2])


# --------------------------------------------------------------------------- helpers

def random_layer(rng, M, K, N, n_out=0, factor=20.0, x_std=1.0, w_std=0.05):
    X = (rng.standard_normal((M, K)) * x_std)
    cols = rng.choice(K, size=n_out, replace=False) if n_out else np.array([], int)
    X[:, cols] *= factor
    W = rng.standard_normal((N, K)) * w_std
    return X.astype(np.float16), W.astype(np.float16), cols


# --------------------------------------------------------------------------- quantizer

@pytest.mark.parametrize("seed", range(4))
def test_quantizer_is_nearest_even_of_float32_quotient(seed):
    """Each q is the nearest integer to fl32(x / s), halves to even, and s = fl32(a/127)."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((6, 64)).astype(np.float16)
    X[0, :8] = np.array([127, 63.5, 2.5, -2.5, 0.5, -1.5, 3.5, 1], np.float16)  # ties, s = 1
    mask, _ = oracle.outlier_columns(X, math.inf)
    Xq, sx = oracle.quantize_rows(X, mask)
    for i in range(X.shape[0]):
        a = np.float32(np.abs(X[i].astype(np.float32)).max())
        assert sx[i] == fl32_div(a, np.float32(127.0))
        for j in range(X.shape[1]):
            v = float(fl32_div(np.float32(X[i, j]), sx[i]))
            q = int(Xq[i, j])
            assert abs(v - q) <= 0.5
            if abs(v - q) == 0.5:
                assert q % 2 == 0
            assert -127 <= q <= 127


def test_weight_quantizer_same_rule_per_output_channel():
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((9, 40)) * 0.03).astype(np.float16)
    W[3] = 0                                           # all-zero channel: scale 0, q 0
    Wq, sw = oracle.quant_weight(W)
    assert sw[3] == 0 and not Wq[3].any()
    for n in range(W.shape[0]):
        if n == 3:
            continue
        a = np.float32(np.abs(W[n].astype(np.float32)).max())
        assert sw[n] == fl32_div(a, np.float32(127.0))
        assert np.abs(Wq[n]).max() == 127              # the absmax element maps to +-127
        for k in range(W.shape[1]):
            v = float(fl32_div(np.float32(W[n, k]), sw[n]))
            assert abs(v - int(Wq[n, k])) <= 0.5


def test_threshold_is_strict_and_over_all_rows():
    X = np.zeros((3, 40), np.float16)
    X[0, 1] = 6.0                                    # equal to t: not an outlier
    X[2, 5] = np.float16(6.0).item() + 0.00390625    # next binary16 above 6: outlier
    X[1, 9] = -7.0                                   # sign does not matter
    X[2, 33] = 100.0                                 # second mask word
    mask, cols = oracle.outlier_columns(X, 6.0)
    np.testing.assert_array_equal(cols, [5, 9, 33])
    assert mask[0] == (1 << 5) | (1 << 9) and mask[1] == (1 << 1)
    # negative thresholds act as 0: every column holding a nonzero value is an outlier
    _, c_neg = oracle.outlier_columns(X, -3.0)
    _, c_zero = oracle.outlier_columns(X, 0.0)
    np.testing.assert_array_equal(c_neg, c_zero)
    np.testing.assert_array_equal(c_zero, [1, 5, 9, 33])
    with pytest.raises(oracle.OracleError):
        oracle.outlier_columns(X, float("nan"))


def test_row_scale_excludes_outlier_columns():
    X = np.array([[1.0, 50.0, -2.0, 0.5], [0.25, -0.125, 0.5, 0.0]], np.float16)
    mask, cols = oracle.outlier_columns(X, 6.0)
    assert list(cols) == [1]
    Xq, sx = oracle.quantize_rows(X, mask)
    assert sx[0] == fl32_div(np.float32(2.0), np.float32(127.0))   # not 50/127
    assert Xq[0, 1] == 0 and Xq[1, 1] == 0
    assert Xq[0, 2] == -127 and Xq[1, 2] == 127


def test_all_outlier_row_and_zero_row():
    X = np.array([[0.0, 0.0, 0.0, 0.0], [9.0, 0.0, -8.0, 0.0]], np.float16)
    mask, cols = oracle.outlier_columns(X, 6.0)
    Xq, sx = oracle.quantize_rows(X, mask)
    assert list(cols) == [0, 2]
    assert sx[0] == 0 and sx[1] == 0 and not Xq.any()


# --------------------------------------------------------------------------- invariants

@pytest.mark.parametrize("seed", range(3))
def test_sign_symmetry(seed):
    rng = np.random.default_rng(10 + seed)
    X, W, _ = random_layer(rng, 5, 48, 7, n_out=2)
    Wq, sw = oracle.quant_weight(W)
    m1, c1 = oracle.outlier_columns(X, 6.0)
    m2, c2 = oracle.outlier_columns(-X, 6.0)
    np.testing.assert_array_equal(c1, c2)
    q1, s1 = oracle.quantize_rows(X, m1)
    q2, s2 = oracle.quantize_rows(-X, m2)
    np.testing.assert_array_equal(q2, -q1)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(oracle.gemm_i32(q2, Wq), -oracle.gemm_i32(q1, Wq))
    Y1 = oracle.linear_forward(X, Wq, sw, None, 6.0)
    Y2 = oracle.linear_forward(-X, Wq, sw, None, 6.0)
    np.testing.assert_array_equal(f16_bits(Y2), f16_bits(-Y1))


@pytest.mark.parametrize("e", [-3, -1, 2, 4])
def test_power_of_two_scaling(e):
    rng = np.random.default_rng(20)
    X, _, _ = random_layer(rng, 4, 64, 1, n_out=3)
    # keep every value a normal binary16 after scaling so that the scaling is exact
    X = (np.sign(X.astype(np.float64)) * np.maximum(np.abs(X.astype(np.float64)), 0.01)).astype(np.float16)
    X2 = (X.astype(np.float64) * 2.0**e).astype(np.float16)
    assert np.array_equal(X2.astype(np.float64), X.astype(np.float64) * 2.0**e)  # exact
    m1, c1 = oracle.outlier_columns(X, 6.0)
    m2, c2 = oracle.outlier_columns(X2, 6.0 * 2.0**e)
    np.testing.assert_array_equal(c1, c2)
    q1, s1 = oracle.quantize_rows(X, m1)
    q2, s2 = oracle.quantize_rows(X2, m2)
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(s2, s1 * np.float32(2.0**e))


def test_column_permutation():
    rng = np.random.default_rng(30)
    X, W, _ = random_layer(rng, 6, 96, 5, n_out=3)
    perm = rng.permutation(96)
    Wq, sw = oracle.quant_weight(W)
    Wq_p, sw_p = oracle.quant_weight(W[:, perm])
    np.testing.assert_array_equal(Wq_p, Wq[:, perm])
    np.testing.assert_array_equal(sw_p, sw)
    m, c = oracle.outlier_columns(X, 6.0)
    mp, cp = oracle.outlier_columns(X[:, perm], 6.0)
    np.testing.assert_array_equal(np.sort(perm[cp]), c)
    q, s = oracle.quantize_rows(X, m)
    qp, sp = oracle.quantize_rows(X[:, perm], mp)
    np.testing.assert_array_equal(qp, q[:, perm])
    np.testing.assert_array_equal(sp, s)
    np.testing.assert_array_equal(oracle.gemm_i32(qp, Wq_p), oracle.gemm_i32(q, Wq))


def test_rows_are_independent_given_the_outlier_set():
    rng = np.random.default_rng(40)
    X, W, _ = random_layer(rng, 9, 64, 6, n_out=2)
    Wq, sw = oracle.quant_weight(W)
    m, _ = oracle.outlier_columns(X, 6.0)
    q, s = oracle.quantize_rows(X, m)
    for i in range(9):
        qi, si = oracle.quantize_rows(X[i:i + 1], m)
        np.testing.assert_array_equal(qi[0], q[i])
        assert si[0] == s[i]
    Y = oracle.linear_forward(X, Wq, sw, None, 6.0)
    rows = [8, 0, 3]
    Yr, Ar = oracle.linear_forward_rows(X, Wq, sw, None, 6.0, rows)
    np.testing.assert_array_equal(f16_bits(Yr), f16_bits(Y[rows]))
    np.testing.assert_array_equal(Ar, oracle.gemm_i32(q, Wq)[rows])


# --------------------------------------------------------------------------- library routines

@pytest.mark.parametrize("shape", [(3, 5, 7), (16, 64, 33), (1, 300, 2)])
def test_int8_product_equals_integer_matmul(shape):
    M, K, N = shape
    rng = np.random.default_rng(K)
    Xq = rng.integers(-127, 128, (M, K), dtype=np.int8)
    Wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
    A = oracle.gemm_i32(Xq, Wq)
    np.testing.assert_array_equal(A, Xq.astype(np.int64) @ Wq.astype(np.int64).T)


def test_int8_product_rejects_int32_overflow():
    K = 133200                      # 127*127*133200 > 2^31 - 1
    Xq = np.full((1, K), 127, np.int8)
    with pytest.raises(oracle.OracleError):
        oracle.gemm_i32(Xq, Xq)
    assert oracle.gemm_i32(Xq[:, :133000], Xq[:, :133000])[0, 0] == 127 * 127 * 133000


def test_threshold_inf_is_pure_vectorwise_int8():
    rng = np.random.default_rng(50)
    X, W, _ = random_layer(rng, 7, 80, 9, n_out=2)
    b = (rng.standard_normal(9) * 0.1).astype(np.float16)
    Wq, sw = oracle.quant_weight(W)
    m, c = oracle.outlier_columns(X, math.inf)
    assert c.size == 0 and not m.any()
    q, s = oracle.quantize_rows(X, m)
    A = q.astype(np.int64) @ Wq.astype(np.int64).T
    ref = (A * s.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
           + b.astype(np.float64)[None, :]).astype(np.float16)
    Y = oracle.linear_forward(X, Wq, sw, b, math.inf)
    np.testing.assert_array_equal(f16_bits(Y), f16_bits(ref))


def test_threshold_zero_is_fp16_matmul_on_rebuilt_weights():
    rng = np.random.default_rng(60)
    X, W, _ = random_layer(rng, 8, 128, 24)
    b = (rng.standard_normal(24) * 0.1).astype(np.float16)
    Wq, sw = oracle.quant_weight(W)
    m, c = oracle.outlier_columns(X, 0.0)
    assert c.size == 128                                  # no all-zero column in X
    q, _ = oracle.quantize_rows(X, m)
    assert not q.any()
    W_hat = (Wq.astype(np.float32) * sw[:, None]).astype(np.float16)     # numpy's own rounding
    np.testing.assert_array_equal(f16_bits(oracle.outlier_weights(Wq, sw, c)), f16_bits(W_hat))
    exact = X.astype(np.float64) @ W_hat.astype(np.float64).T + b.astype(np.float64)
    Y = oracle.linear_forward(X, Wq, sw, b, 0.0).astype(np.float64)
    ref = exact.astype(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert (np.abs(Y - ref) <= ulp).all()
    assert np.mean(Y == ref) > 0.99


# --------------------------------------------------------------------------- error bound

def ulp16(v):
    return np.spacing(np.abs(np.asarray(v, np.float64)).astype(np.float16)).astype(np.float64)


@pytest.mark.parametrize("seed,n_out", [(70, 0), (71, 3), (72, 7)])
def test_error_bound_against_unquantized_product(seed, n_out):
    """|Y - (X W^T + b)| is within the sum of the per-term quantization errors."""
    rng = np.random.default_rng(seed)
    M, K, N = 6, 96, 11
    X, W, _ = random_layer(rng, M, K, N, n_out=n_out, factor=15.0)
    b = (rng.standard_normal(N) * 2.0).astype(np.float16)   # large enough to be noticed
    Wq, sw = oracle.quant_weight(W)
    m, cols = oracle.outlier_columns(X, 6.0)
    assert cols.size == n_out
    q, sx = oracle.quantize_rows(X, m)
    Y = oracle.linear_forward(X, Wq, sw, b, 6.0).astype(np.float64)
    x = X.astype(np.float64)
    w = W.astype(np.float64)
    exact = x @ w.T + b.astype(np.float64)
    is_out = np.zeros(K, bool)
    is_out[cols] = True
    sxd, swd = sx.astype(np.float64), sw.astype(np.float64)
    W_hat = (Wq.astype(np.float32) * sw[:, None]).astype(np.float16).astype(np.float64)
    for i in range(M):
        for n in range(N):
            r = ~is_out
            bound = np.sum(np.abs(x[i, r]) * swd[n] / 2 + np.abs(w[n, r]) * sxd[i] / 2
                           + sxd[i] * swd[n] / 4) * (1 + 1e-5)
            o = is_out
            bound += np.sum(np.abs(x[i, o]) * (swd[n] / 2 + ulp16(W_hat[n, o])))
            bound += ulp16(Y[i, n])
            assert abs(Y[i, n] - exact[i, n]) <= bound, (i, n, Y[i, n], exact[i, n], bound)
