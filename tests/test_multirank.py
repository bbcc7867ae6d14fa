"""Multi-rank logic on CPU: two gloo ranks.

bench.py: ranks tune independent layers (different seeds, no data exchange);
the only cross-rank operation is the MAX of the measured device time, and the
job's throughput is world x steps / max time.

One layer split by output rows: each rank runs the method's step on its rows
with the whole layer's loss normaliser (what ar_tune_step_shard does on a
GPU); the union of the shards' states is the unsharded step's state, bit for
bit, and the SUM of the shards' losses is the layer's loss.
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


# ----------------------------------------------------------------------------
# one layer split by output rows over two ranks (no exchange on the data path)
# ----------------------------------------------------------------------------

def _shard_worker(rank, world, port, bounds, out):
    """Rank r tunes rows bounds[r]:bounds[r+1] of one layer with the oracle's
    step and the whole layer's loss normaliser; the only collective is the
    one-float SUM of the loss, for reporting."""
    import numpy as np

    import synth
    from oracle import autoround_oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        N, K, M, g = bounds[-1], 256, 48, 64
        d = synth.make_linear(N, K, M, seed=17)
        V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
        lo, hi = bounds[rank], bounds[rank + 1]
        Wf = synth.bf16_bits_to_f32(d["W"][lo:hi])
        Xf = synth.bf16_bits_to_f32(d["X"])
        Y = O.reference_forward(Xf, Wf)  # this rank's columns of the reference output
        cfg = O.QConfig(bits=4, group_size=g)
        st = (V[lo:hi], a[lo:hi], b[lo:hi])
        losses = []
        for _ in range(3):
            L, st, _, _ = O.tune_step_linear(Wf, Xf, Y, *st, cfg, count=M * N)
            t = torch.tensor([L], dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.SUM)
            losses.append(float(t.item()))
        out[rank] = (st, losses)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_row_shards_over_two_gloo_ranks_reproduce_the_unsharded_step():
    import numpy as np

    import synth
    from oracle import autoround_oracle as O

    bounds = [0, 24, 64]  # uneven shards: 24/64 is not a power of two
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(2, port, bounds, out), nprocs=2, join=True)
        res = dict(out)
    N, K, M, g = 64, 256, 48, 64
    d = synth.make_linear(N, K, M, seed=17)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    Wf, Xf = synth.bf16_bits_to_f32(d["W"]), synth.bf16_bits_to_f32(d["X"])
    Y = O.reference_forward(Xf, Wf)
    cfg = O.QConfig(bits=4, group_size=g)
    st, ref_losses = (V, a, b), []
    for _ in range(3):
        L, st, _, _ = O.tune_step_linear(Wf, Xf, Y, *st, cfg)
        ref_losses.append(L)
    for i in range(3):  # V, alpha, beta: the shards' rows are the unsharded rows, bit for bit
        joined = np.concatenate([res[0][0][i], res[1][0][i]], axis=0)
        assert np.array_equal(joined, st[i])
    assert res[0][1] == res[1][1]
    assert np.allclose(res[0][1], ref_losses, rtol=1e-12)
