"""The N>1 path of bench.py on CPU with gloo, world_size 2: every rank verifies its own seeded
batch (no data-path collective), times are reduced by max over ranks, and the whole-job rate
counts every rank's tokens.  The per-rank verify step runs on the oracle here (no GPU)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import oracle
import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, seed = bench.rank_workload("tiny", rank)
        inp = W.make_inputs(w, seed=seed, nan_guard=False)
        _, acc, res = oracle.verify_step(inp)
        local_ms = [10.0 + 5.0 * rank, 1.0 + rank]          # rank 1 is the slow one
        mx = bench.reduce_over_ranks(local_ms, world)
        rate = bench.aggregate_rate(bench.tokens_per_step(inp), world, 3, mx[0])
        out[rank] = (seed, int(acc["accept_len"][0]), mx, rate, int(res[2][0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.slow
def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    assert r0[0] != r1[0]                                   # distinct seeds: distinct sequences
    assert r0[2] == r1[2] == [15.0, 2.0]                    # max over ranks, identical on all ranks
    assert r0[3] == r1[3] == pytest.approx(2 * 8 * 3 / 15e-3)
    # each rank's result equals running its shard alone in this process
    for rank, r in ((0, r0), (1, r1)):
        w, seed = bench.rank_workload("tiny", rank)
        _, acc, res = oracle.verify_step(W.make_inputs(w, seed=seed, nan_guard=False))
        assert r[1] == int(acc["accept_len"][0]) and r[4] == int(res[2][0])
