"""The multi-rank path of bench.py on CPU: two gloo ranks (127.0.0.1).

Every rank runs its own replica (weak scaling, no data-path collective); the
only cross-rank steps are the timing reduction (max over ranks) and the
barrier.  This checks both ranks agree on the slowest time, draw different
seeded inputs, and that the whole-job rate counts all ranks' work."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from io_aware_exact_flashattention_b200.inputs import prefill_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 5.0 - rank, 3.0 * (rank + 1)]
        bench.barrier(world)
        got = bench.max_over_ranks(local, world)
        q, _, _ = prefill_inputs(1, 2, 2, 4, 4, 8, bench.rank_seed(7, rank))
        gathered = [torch.zeros_like(q.float()) for _ in range(world)]
        dist.all_gather(gathered, q.float())
        out[rank] = (got, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_seed():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()  # no fork of a threaded process
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        got, same_inputs = out[rank]
        assert got == [11.0, 5.0, 6.0]
        assert not same_inputs  # per-rank seeds give different replicas


def test_aggregate_rate_counts_all_ranks():
    # 2 ranks x 1e12 work x 10 steps in 5 ms (the slowest rank) -> 4e15 / s
    assert bench.aggregate_rate(2, 1e12, 10, 5.0) == pytest.approx(4e15)
    assert bench.aggregate_rate(1, 1e12, 10, 5.0) == pytest.approx(2e15)
