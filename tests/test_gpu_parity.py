"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same inputs.

Small shapes that span several 128 x 256 output tiles with ragged edges are compared in
full; the full-size workloads are compared in full on the integer stages the oracle can
afford (weights, outlier set, activation codes and scales) and on sampled rows for the
int32 accumulators and Y.
"""
import math

import numpy as np
import pytest
import torch

import int8_mixed_precision_absmax_b200 as i8
import oracle
import synth
from tests.gpu_helpers import (assert_y_close, f16_bits, sample_rows, to_dev, to_np,
                               workload_inputs)

pytestmark = pytest.mark.gpu


def run_all_stages(X, W, b, t):
    """Every diagnostic entry point plus the forward, on device; results back on host."""
    Xd, Wd = to_dev(X), to_dev(W)
    bd = None if b is None else to_dev(b)
    Wq, sw = i8.int8_quant_weight(Wd)
    Xq, sx, cols, n = i8.int8_quantize_rows(Xd, t)
    C = i8.int8_gemm_i32(Xq, Wq)
    W_hat = i8.int8_outlier_weights(Wq, sw, cols, n)
    ws = i8.new_workspace(X.shape[0], W.shape[0], X.shape[1], Xd.device)
    Y = i8.int8_linear_forward(Xd, Wq, sw, bd, t, workspace=ws)
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0
    torch.cuda.synchronize()
    k = int(to_np(n)[0])
    return dict(Wq=to_np(Wq), sw=to_np(sw), Xq=to_np(Xq), sx=to_np(sx), cols=to_np(cols)[:k],
                C=to_np(C), W_hat=to_np(W_hat)[:, :k], Y=to_np(Y))


def check_against_oracle_full(X, W, b, t):
    g = run_all_stages(X, W, b, t)
    Wq, sw = oracle.quant_weight(W)
    np.testing.assert_array_equal(g["Wq"], Wq)
    np.testing.assert_array_equal(g["sw"].view(np.uint32), sw.view(np.uint32))
    mask, cols = oracle.outlier_columns(X, t)
    np.testing.assert_array_equal(g["cols"], cols)
    Xq, sx = oracle.quantize_rows(X, mask)
    np.testing.assert_array_equal(g["Xq"], Xq)
    np.testing.assert_array_equal(g["sx"].view(np.uint32), sx.view(np.uint32))
    np.testing.assert_array_equal(g["C"], oracle.gemm_i32(Xq, Wq))
    np.testing.assert_array_equal(f16_bits(g["W_hat"]), f16_bits(oracle.outlier_weights(Wq, sw, cols)))
    Y_ref = oracle.linear_forward(X, Wq, sw, b, t)
    assert_y_close(g["Y"], Y_ref)
    return g, Y_ref


def random_case(M, K, N, n_out, seed, factor=20.0, bias=True):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    cols = rng.choice(K, size=n_out, replace=False) if n_out else []
    X[:, cols] *= factor
    W = rng.standard_normal((N, K)) * 0.02
    b = (rng.standard_normal(N) * 0.01).astype(np.float16) if bias else None
    return X.astype(np.float16), W.astype(np.float16), b


# ------------------------------------------------------------------ small, compared in full

@pytest.mark.parametrize("M,K,N,n_out", [
    (300, 1040, 600, 5),    # ragged in M, N and K (K % 128 != 0), 3 x 3 tiles
    (129, 256, 257, 1),     # one row / one column past a tile
    (16, 256, 256, 2),      # the tiny workload's shape
    (1, 16, 1, 0),          # smallest legal layer
    (8, 4096, 300, 6),      # decode-like rows
    (200, 512, 520, 70),    # more outliers than one 64-wide fp16 block
    (5, 20000, 70, 3),      # rows longer than the register-resident path
])
def test_small_layers_every_stage(M, K, N, n_out):
    X, W, b = random_case(M, K, N, n_out, seed=M * 7 + K + N)
    check_against_oracle_full(X, W, b, 6.0)


def test_tiny_workload_every_stage():
    w, X, W, b, _ = workload_inputs("tiny")
    g, _ = check_against_oracle_full(X, W, b, w.threshold)
    assert list(g["cols"]) == [7, 200]


@pytest.mark.parametrize("t", [math.inf, 0.0, -1.0, 1e-3, 2.5])
def test_thresholds(t):
    X, W, b = random_case(70, 384, 300, 4, seed=3)
    g, _ = check_against_oracle_full(X, W, b, t)
    if t == math.inf:
        assert g["cols"].size == 0
    if t <= 0:
        assert g["cols"].size == 384 and not g["Xq"].any() and not g["C"].any()


def test_zero_rows_and_all_zero_input():
    X, W, b = random_case(40, 256, 64, 2, seed=5)
    X[3] = 0
    X[17] = 0
    check_against_oracle_full(X, W, b, 6.0)
    check_against_oracle_full(np.zeros_like(X), W, b, 6.0)


def test_all_outlier_row_and_zero_weight_channel():
    X, W, b = random_case(12, 128, 40, 0, seed=9)
    X[5, :] = 0
    X[5, 10] = 50.0            # row 5: its only nonzero is an outlier -> scale 0
    W[7] = 0                   # channel 7: scale 0
    check_against_oracle_full(X, W, None, 6.0)


def test_repeated_calls_are_bit_identical():
    X, W, b = random_case(150, 512, 300, 3, seed=11)
    a = run_all_stages(X, W, b, 6.0)
    c = run_all_stages(X, W, b, 6.0)
    for k in a:
        np.testing.assert_array_equal(a[k], c[k])


def test_nan_threshold_and_bad_shape_are_rejected_on_device():
    X = torch.zeros((4, 32), dtype=torch.float16, device="cuda")
    W = torch.zeros((8, 32), dtype=torch.float16, device="cuda")
    Wq, sw = i8.int8_quant_weight(W)
    with pytest.raises(i8.Int8mmError) as e:
        i8.int8_linear_forward(X, Wq, sw, None, float("nan"))
    assert e.value.status == -4
    with pytest.raises(i8.Int8mmError) as e:
        i8.int8_linear_forward(torch.zeros((4, 40), dtype=torch.float16, device="cuda"),
                               torch.zeros((8, 40), dtype=torch.int8, device="cuda"), sw, None)
    assert e.value.status == -3


# ------------------------------------------------------------------ full-size workloads

FULL = ["decode_q_proj", "prefill_up_proj", "down_proj_13b"]


def check_full_size(w, X, W, b, t, n_rows=6, check_weights=True, weights_cache=None):
    Xd = to_dev(X)
    if weights_cache is not None and "Wq" in weights_cache:
        Wq_d, sw_d, Wq, sw = weights_cache["Wq"]
    else:
        Wq_d, sw_d = i8.int8_quant_weight(to_dev(W))
        Wq, sw = to_np(Wq_d), to_np(sw_d)
        if check_weights:
            Wq_ref, sw_ref = oracle.quant_weight(W)
            np.testing.assert_array_equal(Wq, Wq_ref)
            np.testing.assert_array_equal(sw.view(np.uint32), sw_ref.view(np.uint32))
        if weights_cache is not None:
            weights_cache["Wq"] = (Wq_d, sw_d, Wq, sw)
    Xq_d, sx_d, cols_d, n_d = i8.int8_quantize_rows(Xd, t)
    k = int(to_np(n_d)[0])
    mask, cols = oracle.outlier_columns(X, t)
    np.testing.assert_array_equal(to_np(cols_d)[:k], cols)
    Xq, sx = oracle.quantize_rows(X, mask)
    np.testing.assert_array_equal(to_np(Xq_d), Xq)
    np.testing.assert_array_equal(to_np(sx_d).view(np.uint32), sx.view(np.uint32))
    rows = sample_rows(w.M, n_rows)
    C = to_np(i8.int8_gemm_i32(Xq_d, Wq_d))
    ws = i8.new_workspace(w.M, w.N, w.K, Xd.device)
    Y = to_np(i8.int8_linear_forward(Xd, Wq_d, sw_d, None if b is None else to_dev(b), t,
                                     workspace=ws))
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0
    Y_ref, A_ref = oracle.linear_forward_rows(X, Wq, sw, b, t, rows)
    np.testing.assert_array_equal(C[rows], A_ref)
    assert_y_close(Y[rows], Y_ref, f"{w.name} Y[sampled rows]")
    assert np.isfinite(Y.astype(np.float32)).all()
    return cols


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    w, X, W, b, planted = workload_inputs(name)
    cols = check_full_size(w, X, W, b, w.threshold)
    assert set(planted.tolist()) <= set(cols.tolist())


_W175 = {}


@pytest.mark.parametrize("frac,t", [(0.001, 6.0), (0.01, 0.0), (0.01, math.inf)])
def test_full_size_175b(frac, t):
    name = f"ffn_175b_f{frac:g}_t{t:g}"
    w, X, W, b, _ = workload_inputs(name)
    check_full_size(w, X, W, b, t, n_rows=3, check_weights=not _W175, weights_cache=_W175)


@pytest.mark.parametrize("frac", [0.0, 0.001, 0.01])
@pytest.mark.parametrize("t", [0.0, 6.0, math.inf])
def test_175b_sweep_narrow(frac, t):
    """The 175B activation sweep at full M and K with a 2304-channel slice of W."""
    name = f"ffn_175b_f{frac:g}_t{t:g}"
    w, X, W, b, _ = workload_inputs(name, N=2304)
    g_cols = check_full_size(w, X, W, b, t, n_rows=4)
    if t == math.inf:
        assert g_cols.size == 0


# ------------------------------------------------------------------ accumulators and few tokens

def check_forward_acc(X, W, b, t, rows=None):
    """Y and the int32 accumulators of int8_linear_forward_acc against the oracle."""
    Xd = to_dev(X)
    Wq_d, sw_d = i8.int8_quant_weight(to_dev(W))
    ws = i8.new_workspace(X.shape[0], W.shape[0], X.shape[1], Xd.device)
    Y, acc = i8.int8_linear_forward_acc(Xd, Wq_d, sw_d, None if b is None else to_dev(b), t,
                                        workspace=ws)
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0
    Y, acc = to_np(Y), to_np(acc)
    Wq, sw = to_np(Wq_d), to_np(sw_d)
    if rows is None:
        rows = np.arange(X.shape[0])
    Y_ref, A_ref = oracle.linear_forward_rows(X, Wq, sw, b, t, rows)
    np.testing.assert_array_equal(acc[rows], A_ref)
    assert_y_close(Y[rows], Y_ref)
    # the forward without accumulators gives the same Y bits
    Y2 = to_np(i8.int8_linear_forward(Xd, Wq_d, sw_d, None if b is None else to_dev(b), t,
                                      workspace=ws))
    np.testing.assert_array_equal(f16_bits(Y2), f16_bits(Y))
    return Y, acc


@pytest.mark.parametrize("M,K,N,n_out,t", [
    (1, 16, 1, 0, 6.0),
    (1, 4096, 4096, 3, 6.0),
    (3, 1040, 300, 2, 6.0),     # ragged K and N on the few-token path
    (8, 4096, 4096, 6, 6.0),    # the decode shape
    (16, 2048, 640, 5, 6.0),    # the largest few-token batch
    (16, 256, 128, 0, math.inf),
    (7, 512, 384, 0, 0.0),      # every column an outlier: int8 product is zero
    (5, 20000, 200, 4, 6.0),    # long rows: a weight ring that is refilled
    (16, 16384, 300, 4, 6.0),   # activations too long for shared memory: cluster path
    (12, 14336, 256, 3, 6.0),   # cluster path, ragged rows
    (9, 4096, 4100, 5, 6.0),    # channels not a multiple of the per-CTA share
    (17, 512, 300, 3, 6.0),     # one row past the few-token path
    (200, 1040, 600, 5, 6.0),   # the tiled path
    # the one-launch decode kernel (M <= 8, K % 128 == 0, K <= 8192)
    (8, 128, 64, 1, 6.0),       # one k-block: a single slice of the cluster holds X
    (2, 8192, 512, 4, 6.0),     # longest rows: two-box ring, refilled six times
    (6, 3072, 1000, 3, 6.0),    # three boxes, channels not a multiple of 32
    (8, 2176, 96, 2, 6.0),      # 17 k-blocks over 8 slices; most CTAs past N
    (5, 4096, 256, 40, 6.0),    # many outlier columns
    (8, 1024, 1024, 0, 0.0),    # every column an outlier: the fp16 term everywhere
    (4, 512, 96, 0, math.inf),  # no outlier term at all
    (8, 6144, 300, 2, 6.0),     # six boxes through a two-box ring
])
def test_forward_accumulators_and_y(M, K, N, n_out, t):
    X, W, b = random_case(M, K, N, n_out, seed=M + 3 * K + 7 * N)
    Y, acc = check_forward_acc(X, W, b, t)
    if t == 0.0:
        assert not acc.any()


@pytest.mark.parametrize("M,K,N,cols,t", [
    (8, 2048, 512, list(range(640, 704)), 6.0),       # 64 outlier columns in 8 chunks
    (8, 2048, 512, list(range(640, 705)), 6.0),       # 65 columns: a ninth, partial chunk
    (6, 4096, 384, list(range(3, 4096, 57)), 6.0),    # 72 chunks: more than the 64 kept
    (7, 1024, 200, [0, 1, 2, 1023], 6.0),             # first and last columns
])
def test_decode_outlier_term_routes(M, K, N, cols, t):
    """The one-launch decode kernel keeps the fp16 activations of up to 64 chunks of 8 columns
    that hold an outlier in shared memory and reads the others from X again; the fp16 term runs
    on the warp-level fp16 MMA either way.  Both cases against the oracle."""
    rng = np.random.default_rng(M * K + N + len(cols))
    X = rng.standard_normal((M, K))
    X[:, cols] *= rng.uniform(10, 40, size=len(cols))
    X[0, cols] = rng.uniform(20, 40, size=len(cols)) * rng.choice([-1, 1], size=len(cols))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    b = (rng.standard_normal(N) * 0.01).astype(np.float16)
    X = X.astype(np.float16)
    _, found = oracle.outlier_columns(X, t)
    np.testing.assert_array_equal(found, np.array(sorted(cols)))
    check_forward_acc(X, W, b, t)


def test_decode_workload_full_forward():
    w, X, W, b, _ = workload_inputs("decode_q_proj")
    Y, acc = check_forward_acc(X, W, b, w.threshold)
    # repeated calls: same bits every time
    Y2, acc2 = check_forward_acc(X, W, b, w.threshold)
    np.testing.assert_array_equal(acc, acc2)
    np.testing.assert_array_equal(f16_bits(Y), f16_bits(Y2))


def test_few_token_path_many_calls_one_workspace():
    X, W, b = random_case(8, 1024, 1024, 3, seed=21)
    Xd = to_dev(X)
    Wq_d, sw_d = i8.int8_quant_weight(to_dev(W))
    ws = i8.new_workspace(8, 1024, 1024, Xd.device)
    first = to_np(i8.int8_linear_forward(Xd, Wq_d, sw_d, to_dev(b), 6.0, workspace=ws))
    Ys = [i8.int8_linear_forward(Xd, Wq_d, sw_d, to_dev(b), 6.0, workspace=ws) for _ in range(50)]
    torch.cuda.synchronize()
    for Y in Ys:
        np.testing.assert_array_equal(f16_bits(to_np(Y)), f16_bits(first))
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0


@pytest.mark.parametrize("M", [4, 16, 40])
def test_quantizer_ties_and_near_ties_exact(M):
    """Values placed on and next to half-integer quotients; W = I makes acc = 127 * Xq."""
    K = 256
    rng = np.random.default_rng(100 + M)
    X = rng.standard_normal((M, K)) * 0.05
    for i in range(M):
        a = float(np.float16(1.0029296875 + 0.0078125 * i))  # row absmax
        X[i, 0] = a
        ks = rng.integers(-126, 126, size=120)
        X[i, 1:121] = (ks + 0.5) * a / 127.0           # lands on or near x/s = k + 1/2
    X[0, 1] = 0.50146484375                            # the golden division-by-scale case
    X[0, 0] = 1.0029296875
    X = X.astype(np.float16)
    W = np.eye(K, dtype=np.float16)
    Y, acc = check_forward_acc(X, W, None, math.inf)
    Wq, sw = oracle.quant_weight(W)
    assert (np.diag(Wq) == 127).all()
    mask, _ = oracle.outlier_columns(X, math.inf)
    Xq, _ = oracle.quantize_rows(X, mask)
    np.testing.assert_array_equal(acc, 127 * Xq.astype(np.int32))
    assert Xq[0, 1] == 63


@pytest.mark.parametrize("M,K,N", [(8, 4096, 1024), (16, 2048, 512), (64, 512, 520)])
def test_weights_quantized_just_before_the_forward(M, K, N):
    """int8_quant_weight immediately followed by the forward on one stream, with nothing
    launched in between (buffers allocated up front), twice with different weights written into
    the same Wq buffer: the forward (whose decode route starts reading Wq before its dependency
    wait) must see the new weights each time."""
    rng = np.random.default_rng(M + K + N)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, size=3, replace=False)] *= 25.0
    X = X.astype(np.float16)
    Ws = [(rng.standard_normal((N, K)) * s).astype(np.float16) for s in (0.02, 0.05)]
    Xd = to_dev(X)
    Wds = [to_dev(W) for W in Ws]
    Wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    Ys = [torch.empty((M, N), dtype=torch.float16, device="cuda") for _ in Ws]
    ws = i8.new_workspace(M, N, K, Xd.device)
    torch.cuda.synchronize()
    for Wd, Y in zip(Wds, Ys):
        i8.int8_quant_weight(Wd, Wq=Wq, w_scale=sw)
        i8.int8_linear_forward(Xd, Wq, sw, None, 6.0, Y=Y, workspace=ws)
    torch.cuda.synchronize()
    assert i8.int8_read_device_status(ws[:4].view(torch.int32)) == 0
    for W, Y in zip(Ws, Ys):
        Wq_ref, sw_ref = oracle.quant_weight(W)
        assert_y_close(to_np(Y), oracle.linear_forward(X, Wq_ref, sw_ref, None, 6.0))
