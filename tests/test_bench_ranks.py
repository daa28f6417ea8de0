"""The bench's multi-rank plumbing (replicas, max over ranks) on CPU with
two gloo ranks: the slowest rank's time decides, and the whole-job
throughput counts every rank's tokens."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.rank_barrier(world)
        mine = 1.5 + rank  # rank 1 is the slow one
        results[rank] = bench.rank_max(mine, world, "cpu")
        bench.rank_barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    import bench  # noqa: F401  (importable without a GPU)
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world, start_method="spawn")
    assert dict(results) == {0: 2.5, 1: 2.5}


def test_replica_throughput_counts_every_rank():
    import bench
    assert bench.replica_tokens_per_s(1, 4096, 0.5) == pytest.approx(8192000.0)
    assert bench.replica_tokens_per_s(8, 4096, 0.5) == pytest.approx(8 * 8192000.0)
    assert bench.rank_max(3.0, 1, "cpu") == 3.0
