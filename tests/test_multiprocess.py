"""The bench's multi-rank aggregation on CPU with two gloo ranks (replicas: no data-path collective).

Every rank reports its own device time; the job's time is the maximum over ranks and its
throughput counts every rank's bytes. Run as two processes on 127.0.0.1.
"""
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


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    my_ms = [12.5, 20.0][rank]  # rank 1 is the slow replica
    got = bench.max_over_ranks(my_ms)
    results[rank] = (got, bench.job_throughput(1_000_000_000, world, got / 10))
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    world = 2
    with mp.get_context("spawn").Manager() as m:  # no fork of this (multi-threaded) process
        results = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        res = dict(results)
    for rank in range(world):
        ms, gbs = res[rank]
        assert ms == 20.0  # both ranks see the slowest time
        assert abs(gbs - 2 * 1e9 / 2e-3 / 1e9) < 1e-6  # 2 ranks x 1 GB per 2 ms step


def test_single_process_is_its_own_max():
    import bench
    assert bench.max_over_ranks(7.0) == 7.0
    assert bench.job_throughput(2_000_000_000, 1, 1.0) == pytest.approx(2000.0)
