"""The token split of the layer across ranks (rowparallel.py), on CPU with two gloo ranks: the
oracle stands in for each rank's kernels (the forward, the weight quantization and the column
maxima), and the ranks' rows of Y, put back in order, must equal the whole layer's oracle Y bit
for bit.  The planted outlier columns are large in one rank's rows only, so a rank that found
its outlier columns from its own rows alone would get other codes; the test checks that too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from int8_mixed_precision_absmax_b200 import rowparallel as rp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_quantize(w):
    Wq, sw = oracle.quant_weight(w.numpy())
    return torch.from_numpy(Wq), torch.from_numpy(sw)


def _oracle_forward(X, Wq, sw, b, t):
    return torch.from_numpy(oracle.linear_forward(X.numpy(), Wq.numpy(), sw.numpy(),
                                                  None if b is None else b.numpy(), t))


def _oracle_column_absmax(X):
    return torch.from_numpy(np.asarray(oracle.activation_stats(X.numpy())[3], np.float32))


def _numpy_outlier_row(col, t):
    """The appended row, restated for the CPU ranks: col[j] where it exceeds max(t, 0)."""
    c = col.numpy().astype(np.float32)
    return torch.from_numpy(np.where(c > max(float(t), 0.0), c, 0.0).astype(np.float16))


def _layer(M, K, N, split, with_bias, seed):
    """X whose outlier columns are large only in the rows of the second rank."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    cols = rng.choice(K, size=3, replace=False)
    if split < M:
        X[split:, cols] *= 30.0
    X[min(split, M - 1), cols[0]] = 0.0  # not every row of the column is large
    W = rng.standard_normal((N, K)) * 0.05
    b = (rng.standard_normal(N) * 0.1).astype(np.float16) if with_bias else None
    return X.astype(np.float16), W.astype(np.float16), b


def _worker(rank, world, port, M, K, N, split, t, with_bias, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, W, b = _layer(M, K, N, split, with_bias, M + K + N)
        rows = X[:split] if rank == 0 else X[split:]
        layer = rp.RowParallelInt8Linear(torch.from_numpy(W),
                                         None if b is None else torch.from_numpy(b), t,
                                         local_forward=_oracle_forward,
                                         quantize=_oracle_quantize,
                                         column_absmax=_oracle_column_absmax,
                                         outlier_row=_numpy_outlier_row)
        Y = layer(torch.from_numpy(np.ascontiguousarray(rows)).reshape(rows.shape[0], 1, K))
        assert tuple(Y.shape) == (rows.shape[0], 1, N)
        out[rank] = Y.reshape(rows.shape[0], N).numpy().view(np.uint16).tobytes()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M,K,N,split,t,with_bias", [
    (6, 64, 40, 3, 6.0, True),
    (5, 128, 33, 1, 6.0, False),
    (4, 32, 16, 0, 6.0, True),       # the first rank has no rows at all
    (7, 64, 24, 4, float("inf"), True),
    (5, 64, 24, 2, -1.0, False),     # a negative threshold acts as 0
])
def test_two_ranks_give_the_whole_layers_rows(M, K, N, split, t, with_bias):
    world = 2
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), M, K, N, split, t, with_bias, out),
             nprocs=world, join=True)
    X, W, b = _layer(M, K, N, split, with_bias, M + K + N)
    Wq, sw = oracle.quant_weight(W)
    Y_ref = oracle.linear_forward(X, Wq, sw, b, t)
    got = np.concatenate([np.frombuffer(out[r], np.uint16).reshape(-1, N) for r in range(world)])
    np.testing.assert_array_equal(got, Y_ref.view(np.uint16))
    if 0 < split < M and t == 6.0:
        # the first rank alone would have missed the outlier columns
        Y_local = oracle.linear_forward(X[:split], Wq, sw, b, t)
        assert not np.array_equal(Y_local.view(np.uint16), Y_ref[:split].view(np.uint16))
