"""The output-channel split of the layer across ranks (colparallel.py), on CPU with two gloo
ranks: the oracle stands in for each rank's local kernels, and the joined Y must equal the
whole layer's oracle Y bit for bit (every output channel is computed from X and its own weight
row only, so the split changes no arithmetic)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from int8_mixed_precision_absmax_b200 import colparallel as cp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_plan_shards_cover_every_channel_once():
    for n in (1, 15, 16, 17, 300, 4096, 11008):
        for world in (1, 2, 3, 4, 8):
            sh = cp.plan_shards(n, world)
            assert all(s.width % 16 == 0 and s.width == sh[0].width for s in sh)
            covered = [c for s in sh for c in range(s.lo, s.hi)]
            assert covered == list(range(n))
            assert all(0 <= s.real <= s.width for s in sh)


def _oracle_quantize(w):
    Wq, sw = oracle.quant_weight(w.numpy())
    return torch.from_numpy(Wq), torch.from_numpy(sw)


def _oracle_forward(X, Wq, sw, b, t):
    return torch.from_numpy(oracle.linear_forward(X.numpy(), Wq.numpy(), sw.numpy(),
                                                  None if b is None else b.numpy(), t))


def _worker(rank, world, port, M, K, N, with_bias, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(M + K + N)
        X = rng.standard_normal((M, K))
        X[:, rng.choice(K, size=3, replace=False)] *= 30.0
        W = rng.standard_normal((N, K)) * 0.05
        b = (rng.standard_normal(N) * 0.1).astype(np.float16) if with_bias else None
        X, W = X.astype(np.float16), W.astype(np.float16)
        layer = cp.ColumnParallelInt8Linear(torch.from_numpy(W),
                                            None if b is None else torch.from_numpy(b), 6.0,
                                            local_forward=_oracle_forward,
                                            quantize=_oracle_quantize)
        Y = layer(torch.from_numpy(X).reshape(M, 1, K))
        out[rank] = Y.reshape(M, N).numpy().view(np.uint16).tobytes()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M,K,N,with_bias", [(5, 64, 40, True), (3, 128, 300, False),
                                             (1, 32, 16, True)])
def test_two_ranks_join_to_the_whole_layer(M, K, N, with_bias):
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), M, K, N, with_bias, out), nprocs=world, join=True)
    rng = np.random.default_rng(M + K + N)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, size=3, replace=False)] *= 30.0
    W = rng.standard_normal((N, K)) * 0.05
    b = (rng.standard_normal(N) * 0.1).astype(np.float16) if with_bias else None
    X, W = X.astype(np.float16), W.astype(np.float16)
    Wq, sw = oracle.quant_weight(W)
    Y_ref = oracle.linear_forward(X, Wq, sw, b, 6.0)
    for r in range(world):
        got = np.frombuffer(out[r], np.uint16).reshape(M, N)
        np.testing.assert_array_equal(got, Y_ref.view(np.uint16))
