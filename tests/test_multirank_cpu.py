"""The bench's multi-rank host logic on CPU: two gloo ranks, each owning an
independent sequence batch (weak scaling, no data-path collective); the
whole-job throughput uses the max elapsed time over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape = workloads.WORKLOADS["tiny_cca_fp32"]
        mine = bench.rank_workload(shape, rank)
        x = workloads.make_inputs(mine)["x"]

        def reduce_max(v):
            t = torch.tensor([v], dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())

        elapsed = 10.0 + 5.0 * rank  # rank 1 is the slow one
        value, ms = bench.aggregate(elapsed, mine.tokens, 5, world, reduce_max)
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine.seed, float(x.sum())))
        q.put((rank, value, ms, gathered))
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shape = workloads.WORKLOADS["tiny_cca_fp32"]
    for rank, value, ms, gathered in res:
        assert ms == pytest.approx(15.0 / 5)                   # max over ranks
        assert value == pytest.approx(shape.tokens * world / (ms / 1e3))
        seeds = [g[0] for g in gathered]
        assert len(set(seeds)) == world                         # independent batches
        assert gathered[0][1] != gathered[1][1]
