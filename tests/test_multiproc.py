"""bench.py's multi-process plumbing on CPU: two gloo ranks, max over ranks, whole-job rate."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.init_dist(world, "gloo")
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(torch.device("cpu"))
    # each rank timed a different duration; every rank must see the slowest one
    m = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
    out[rank] = m
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_with_gloo(world):
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert dict(out) == {r: 1.5 + world - 1 for r in range(world)}


def test_whole_job_rate_counts_every_rank():
    # 2 ranks x 10 steps x 1e9 ops in 2 s of the slowest rank
    assert bench.whole_job_rate(1e9, 10, 2, 2.0) == pytest.approx(1e10)
    assert bench.max_over_ranks(3.0, torch.device("cpu")) == 3.0  # no process group


def test_reference_arm_on_other_ranks_exits_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1"]) == 0
    assert capsys.readouterr().out == ""
