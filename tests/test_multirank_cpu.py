"""The bench's multi-rank accounting on two CPU ranks (gloo): each rank times
its own batch, the job time is the max over ranks and the work is summed.
No GPU is involved."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from long_context_misa_b200 import inputs as G


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r timed 10 steps in (r + 1) * 5 ms; every rank did 1000 units per step
        out = bench.aggregate((rank + 1) * 5.0, 10, 1000.0, 8, world, dist, "cpu")
        # rank-seeded inputs differ between ranks (independent batches)
        wl = G.WORKLOADS["tiny_decode"]
        first = float(G.make_inputs(wl, seed=rank).q[0, 0, 0])
        gathered = [None] * world
        dist.all_gather_object(gathered, first)
        q.put((rank, out, gathered))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (ms, value, qps), gathered in res:
        assert ms == pytest.approx(1.0)               # max over ranks: 10 ms / 10 steps
        assert value == pytest.approx(2 * 1000.0 / 1e-3)
        assert qps == pytest.approx(2 * 8 / 1e-3)
        assert gathered[0] != gathered[1]             # different batches per rank


def test_single_rank_needs_no_process_group():
    ms, value, qps = bench.aggregate(20.0, 10, 500.0, 4, 1)
    assert ms == pytest.approx(2.0) and value == pytest.approx(500.0 / 2e-3) and qps == pytest.approx(4 / 2e-3)
