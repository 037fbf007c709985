"""The benchmark's multi-rank host logic on CPU with the gloo backend
(world size 2): timings are reduced to the max over ranks, the whole-job rate
divides every rank's units by the slowest rank's time, and only rank 0 runs the
reference arm.  The path itself has no exchange step: ranks are replicas."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [1.0 + rank, 10.0 - rank, 5.0]
        got = bench.max_over_ranks(mine, world)
        rate = bench.aggregate_rate(1e9, world, got[0])

        class A:
            workload = "cfg1"
            override = None
            steps = 1
            warmup = 0
            step_budget = 0.2
        line = bench.run_reference(A(), rank)
        q.put((rank, got, rate, line is None))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank0_only_reference():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = {}
    while not q.empty():
        r, got, rate, ref_none = q.get()
        res[r] = (got, rate, ref_none)
    assert set(res) == {0, 1}
    for r in range(world):
        got, rate, _ = res[r]
        assert got == [2.0, 10.0, 5.0]                         # element-wise max over the ranks
        assert rate == pytest.approx(2 * 1e9 / 2.0e-3)         # all ranks' units / slowest time
    assert res[0][2] is False and res[1][2] is True             # reference arm: rank 0 only
