"""The token split with the library's kernels on the GPU: one NCCL rank (the runs here have one
GPU), so the all-reduce is a copy, but the rank runs the whole path: the column maxima from the
statistics kernel, their MAX all-reduce, the appended outlier row and the forward on the rows
plus that row.  8 rows become 9 (the two-launch few-token path), 40 become 41 (the tiled path);
Y of the real rows is compared with the oracle of the whole layer."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import int8_mixed_precision_absmax_b200 as i8
import oracle
from int8_mixed_precision_absmax_b200 import rowparallel as rp
from tests.gpu_helpers import assert_y_close, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda:0"))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("M,K,N", [(8, 4096, 4096), (40, 1024, 300)])
def test_one_rank_token_split_equals_the_layer(nccl_group, M, K, N):
    rng = np.random.default_rng(3 * M + K + N)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, size=4, replace=False)] *= 30.0
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    b = (rng.standard_normal(N) * 0.01).astype(np.float16)
    X = X.astype(np.float16)
    layer = rp.RowParallelInt8Linear(to_dev(W), to_dev(b), 6.0)
    Y = to_np(layer(to_dev(X)))
    assert Y.shape == (M, N)
    Y_ref = oracle.linear_forward(X, to_np(layer.Wq), to_np(layer.w_scale), b, 6.0)
    assert_y_close(Y, Y_ref, f"token split {M}x{K}x{N}")


def test_outlier_row_marks_exactly_the_columns_above_the_threshold():
    # column maxima are binary16 magnitudes: 6 and its two binary16 neighbours
    col = torch.tensor([0.0, 5.99609375, 6.0, 6.00390625, 60.0, 65504.0] + [1.0] * 10,
                       dtype=torch.float32, device="cuda")
    row = i8.int8_outlier_row(col, 6.0)
    assert row.dtype == torch.float16
    np.testing.assert_array_equal(to_np(row.float())[:6], [0, 0, 0, 6.00390625, 60, 65504])
    assert not to_np(row.float())[6:].any()
    # the kernels see the row exceed the threshold exactly in the marked columns
    np.testing.assert_array_equal(to_np(row.float()) > 6.0, to_np(col) > 6.0)
    assert not to_np(i8.int8_outlier_row(col, float("inf")).float()).any()
    np.testing.assert_array_equal(to_np(i8.int8_outlier_row(col, -3.0).float()), to_np(col))
    with pytest.raises(i8.Int8mmError):
        i8.int8_outlier_row(col, float("nan"))
