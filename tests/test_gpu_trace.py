"""The forward's own intermediates against the oracle, bit for bit, on every dispatch route.

int8_linear_forward_trace returns what the kernels that produce Y computed on the way: the
outlier columns, the row scales, the int8 codes and the fp16 outlier weights.  On the few-token
routes (the one-launch decode kernel, the two-launch few-token pair, the cluster kernel) these
never reach memory on the normal path, so this is where their row scales and codes are checked
bit for bit; on the tiled route they are the workspace regions the product reads.  Y and the
int32 products must equal those of int8_linear_forward_ex bit for bit (same kernels).
"""
import math

import numpy as np
import pytest
import torch

import int8_mixed_precision_absmax_b200 as i8
import oracle
from tests.gpu_helpers import assert_y_close, f16_bits, to_dev, to_np, workload_inputs

pytestmark = pytest.mark.gpu


def random_case(M, K, N, n_out, seed, factor=20.0, bias=True):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    cols = rng.choice(K, size=n_out, replace=False) if n_out else []
    X[:, cols] *= factor
    W = rng.standard_normal((N, K)) * 0.02
    b = (rng.standard_normal(N) * 0.01).astype(np.float16) if bias else None
    return X.astype(np.float16), W.astype(np.float16), b


def check_trace(X, W, b, t, per_tensor=False, keep_w16=False, pair_tiles=False):
    """Every output of the trace against the oracle; returns the trace (host arrays)."""
    Xd = to_dev(X)
    Wd = to_dev(W)
    bd = None if b is None else to_dev(b)
    Wq_d, sw_d = i8.int8_quant_weight(Wd)
    W16 = Wd if keep_w16 else None
    M, K = X.shape
    N = W.shape[0]
    ws = i8.new_workspace(M, N, K, Xd.device)
    tr = i8.int8_linear_forward_trace(Xd, Wq_d, sw_d, bd, t, W16=W16, per_tensor=per_tensor,
                                      workspace=ws, pair_tiles=pair_tiles)
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0
    g = {k: to_np(v) for k, v in tr.items()}
    Wq, sw = to_np(Wq_d), to_np(sw_d)

    # outlier set
    mask, cols = oracle.outlier_columns(X, t)
    n = int(g["n_outliers"][0])
    np.testing.assert_array_equal(g["outlier_cols"][:n], cols)
    # codes and scales
    Xq_ref, sx_ref = (oracle.quantize_tensor if per_tensor else oracle.quantize_rows)(X, mask)
    np.testing.assert_array_equal(g["Xq"], Xq_ref)
    np.testing.assert_array_equal(g["row_scale"].view(np.uint32), sx_ref.view(np.uint32))
    # the fp16 weights the outlier term used
    if len(cols):
        W_used = W[:, cols] if keep_w16 else oracle.outlier_weights(Wq, sw, cols)
        np.testing.assert_array_equal(f16_bits(g["W_hat"][:, cols]), f16_bits(W_used))
    # int32 products and Y
    rows = np.arange(M)
    Y_ref, A_ref = oracle.linear_forward_rows_ex(X, Wq, sw, b, t, rows,
                                                 W16=W if keep_w16 else None,
                                                 per_tensor=per_tensor)
    np.testing.assert_array_equal(g["acc"], A_ref)
    assert_y_close(g["Y"], Y_ref)
    # the same bits as the forward without the trace
    acc2 = torch.empty((M, N), dtype=torch.int32, device=Xd.device)
    Y2 = i8.int8_linear_forward_ex(Xd, Wq_d, sw_d, bd, t, W16=W16, per_tensor=per_tensor,
                                   acc=acc2, workspace=ws, pair_tiles=pair_tiles)
    np.testing.assert_array_equal(f16_bits(to_np(Y2)), f16_bits(g["Y"]))
    np.testing.assert_array_equal(to_np(acc2), g["acc"])
    return g


SHAPES = [
    # (M, K, N, planted outlier columns, threshold)  -- route
    (1, 4096, 4096, 3, 6.0),      # decode kernel
    (8, 4096, 4096, 6, 6.0),      # decode kernel, the decode shape
    (8, 128, 64, 1, 6.0),         # decode kernel, one k-block
    (2, 8192, 512, 4, 6.0),       # decode kernel, longest rows
    (6, 3072, 1000, 3, 6.0),      # decode kernel, channels not a multiple of 32
    (5, 4096, 256, 40, 6.0),      # decode kernel, many outlier columns
    (8, 1024, 1024, 0, 0.0),      # decode kernel, every column an outlier
    (4, 512, 96, 0, math.inf),    # decode kernel, no outlier term
    (16, 2048, 640, 5, 6.0),      # few-token pair
    (9, 4096, 4100, 5, 6.0),      # few-token pair, ragged channels
    (16, 256, 128, 0, math.inf),  # few-token pair, no outliers
    (12, 1024, 256, 0, 0.0),      # few-token pair, every column an outlier
    (1, 16, 1, 0, 6.0),           # cluster kernel, smallest layer
    (3, 1040, 300, 2, 6.0),       # cluster kernel, ragged K
    (16, 16384, 300, 4, 6.0),     # cluster kernel, long rows
    (12, 14336, 256, 3, 6.0),     # cluster kernel, ragged rows
    (5, 20000, 200, 4, 6.0),      # cluster kernel, refilled weight ring
    (17, 512, 300, 3, 6.0),       # tiled path, one row past the few-token routes
    (200, 1040, 600, 5, 6.0),     # tiled path, ragged tiles
    (70, 384, 300, 0, 0.0),       # tiled path, every column an outlier
    (40, 65536, 64, 7, 6.0),      # tiled path, the longest rows: one 128 KB row stage per block
    (33, 24576, 96, 5, 6.0),      # tiled path, rows longer than 16K columns, ragged row groups
    (23, 64, 40, 1, 6.0),         # tiled path, one warp per row (eight rows per block)
    (41, 6144, 96, 4, 6.0),       # tiled path, 128 threads per row (two rows per block)
]


@pytest.mark.parametrize("M,K,N,n_out,t", SHAPES)
def test_trace_every_route(M, K, N, n_out, t):
    X, W, b = random_case(M, K, N, n_out, seed=M + 3 * K + 7 * N)
    check_trace(X, W, b, t)


@pytest.mark.parametrize("M,K,N,n_out,t", [s for s in SHAPES if s[4] == 6.0][::2])
def test_trace_per_tensor_scale(M, K, N, n_out, t):
    X, W, b = random_case(M, K, N, n_out, seed=11 * M + K + N)
    X[M // 2] *= 0.25  # rows of different magnitude: the tensor scale is not every row's own
    check_trace(X, W, b, t, per_tensor=True)


@pytest.mark.parametrize("M,K,N,n_out,t", [s for s in SHAPES if s[4] == 6.0][1::2])
def test_trace_kept_fp16_weights(M, K, N, n_out, t):
    X, W, b = random_case(M, K, N, n_out, seed=13 * M + K + N)
    check_trace(X, W, b, t, keep_w16=True)


@pytest.mark.parametrize("name", ["tiny", "decode_q_proj"])
def test_trace_workloads(name):
    w, X, W, b, planted = workload_inputs(name)
    g = check_trace(X, W, b, w.threshold)
    n = int(g["n_outliers"][0])
    assert set(planted.tolist()) <= set(g["outlier_cols"][:n].tolist())


@pytest.mark.parametrize("M,K", [(4, 256), (8, 1024), (13, 2048), (16, 256), (40, 256),
                                 (3, 1040)])
def test_trace_planted_ties(M, K):
    """Values on and next to half-integer quotients x / s = k + 1/2, on every route: there the
    codes of the IEEE quotient differ from those of the uncorrected product x * RN(1/s), and
    the kernels must give the former."""
    rng = np.random.default_rng(100 + M + K)
    X = rng.standard_normal((M, K)) * 0.05
    for i in range(M):
        a = float(np.float16(1.0029296875 + 0.0078125 * i))  # the row absmax
        X[i, 0] = a
        ks = rng.integers(-126, 126, size=120)
        X[i, 1:121] = (ks + 0.5) * a / 127.0
    X[0, 0] = 1.0029296875
    X[0, 1] = 0.50146484375                                   # a / 2: the exact quotient is 63.5
    X = X.astype(np.float16)
    W = (rng.standard_normal((64, K)) * 0.02).astype(np.float16)
    check_trace(X, W, None, 6.0)


@pytest.mark.parametrize("M,K,N,n_out,t", [
    (300, 1040, 600, 5, 6.0),     # ragged pair tiles in M, N and K
    (129, 256, 257, 1, 6.0),      # one row past a single tile: a pair tile mostly empty
    (512, 2048, 1000, 70, 6.0),   # more outliers than one fp16 k-block
    (384, 512, 520, 0, math.inf), # no outlier term: two accumulator slots
    (256, 384, 300, 0, 0.0),      # every column an outlier: fp16 product only
])
def test_trace_pair_tiles(M, K, N, n_out, t):
    """The products on CTA pairs (256 x 256 tiles, tcgen05 cta_group::2) against the oracle, and
    against the single-CTA tiles bit for bit in the integer stages."""
    X, W, b = random_case(M, K, N, n_out, seed=5 * M + K + N)
    g = check_trace(X, W, b, t, pair_tiles=True)
    g1 = check_trace(X, W, b, t)
    np.testing.assert_array_equal(g["acc"], g1["acc"])


def test_pair_tiles_full_size_prefill():
    w, X, W, b, _ = workload_inputs("prefill_up_proj")
    Xd, Wd = to_dev(X), to_dev(W)
    Wq_d, sw_d = i8.int8_quant_weight(Wd)
    bd = to_dev(b)
    ws = i8.new_workspace(w.M, w.N, w.K, Xd.device)
    acc_p = torch.empty((w.M, w.N), dtype=torch.int32, device="cuda")
    acc_1 = torch.empty((w.M, w.N), dtype=torch.int32, device="cuda")
    Yp = i8.int8_linear_forward_ex(Xd, Wq_d, sw_d, bd, w.threshold, acc=acc_p, workspace=ws,
                                   pair_tiles=True)
    Y1 = i8.int8_linear_forward_ex(Xd, Wq_d, sw_d, bd, w.threshold, acc=acc_1, workspace=ws)
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0
    assert torch.equal(acc_p, acc_1)
    rows = np.array([0, 1, 777, w.M - 1])
    Y_ref, A_ref = oracle.linear_forward_rows(X, to_np(Wq_d), to_np(sw_d), b, w.threshold, rows)
    np.testing.assert_array_equal(to_np(acc_p)[rows], A_ref)
    assert_y_close(to_np(Yp)[rows], Y_ref)
    assert_y_close(to_np(Yp), to_np(Y1))
