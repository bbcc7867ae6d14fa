"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

Ranks tune independent layers (different seeds, no data exchange); the only
cross-rank operation is the MAX of the measured device time, and the job's
throughput is world x steps / max time.
"""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        job_ms = bench.max_over_ranks(local_ms, dist, "cpu")
        seed = bench.rank_seed(0, rank)
        out[rank] = (job_ms, seed, bench.job_throughput(world, 20, job_ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_distinct_layers():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] != res[1][1]
    assert res[0][2] == pytest.approx(2 * 20 / 0.015)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_throughput(1, 10, 100.0) == pytest.approx(100.0)
