"""The output-channel split with the library's kernels on the GPU: one NCCL rank (the runs
here have one GPU), so the gather is a copy, but the rank runs the whole path: its slice of
the weights quantized and multiplied by the kernels, joined by all_gather_into_tensor."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import int8_mixed_precision_absmax_b200 as i8
import oracle
from int8_mixed_precision_absmax_b200 import colparallel as cp
from tests.gpu_helpers import assert_y_close, f16_bits, to_dev, to_np

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
def test_one_rank_split_equals_the_layer(nccl_group, M, K, N):
    rng = np.random.default_rng(M + K + N)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, size=4, replace=False)] *= 30.0
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    b = (rng.standard_normal(N) * 0.01).astype(np.float16)
    X = X.astype(np.float16)
    layer = cp.ColumnParallelInt8Linear(to_dev(W), to_dev(b), 6.0)
    Y = to_np(layer(to_dev(X)))
    Wq, sw = i8.int8_quant_weight(to_dev(W))
    Y_one = to_np(i8.int8_linear_forward(to_dev(X), Wq, sw, to_dev(b), 6.0))
    Y_ref = oracle.linear_forward(X, to_np(Wq), to_np(sw), b, 6.0)
    assert_y_close(Y, Y_ref, f"split {M}x{K}x{N}")
    if N % 16 == 0:  # no padded channels: the same launches as the unsplit layer
        np.testing.assert_array_equal(f16_bits(Y), f16_bits(Y_one))
