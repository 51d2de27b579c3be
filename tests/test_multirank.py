"""The N > 1 host path on CPU: two gloo ranks run independent replicas, the
timing is the max over ranks, and the job's throughput counts every rank's bytes."""

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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        # each rank reports a different step time; the job uses the slowest
        my_ms = [1.0 + rank, 0.5 * (rank + 1)]
        got = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
        value, slowest = bench.job_throughput(4e9, [got[0]] * world)
        results[rank] = (got, value, slowest)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_replicas_max_over_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    for rank in range(world):
        got, value, slowest = res[rank]
        assert got == [2.0, 1.0]                     # max over ranks, element-wise
        assert slowest == 2.0
        assert value == pytest.approx(4e9 * 2 / 2e-3 / 1e9)   # both ranks' bytes over the slowest time


def test_job_throughput_single_rank():
    v, s = bench.job_throughput(5.37e9, [1.0])
    assert s == 1.0 and v == pytest.approx(5370.0)
