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


# ---------------------------------------------------------------- KV-group split --
# One sequence's heads split over two ranks ("Compressed Convolutional Attention",
# gist.science/es/paper/2510.04476, section 2.C: K/V heads shared inside the latent by groups of query
# heads; section 2.B item 2: the QK-mean pairs a query head only with its own group). Each rank runs
# the oracle's block on its KV groups alone, with the value shift splitting the whole block's V
# channels (section 2.B item 3), and the partial outputs summed over the ranks (one all-reduce of y)
# give the whole block's y. The slicing below is this test's own, not the library's.
def _share(inp, nq, nkv, d, rank, world):
    G = nq // nkv
    gk = nkv // world
    k0, k1 = rank * gk * d, (rank + 1) * gk * d
    q0, q1 = rank * gk * G * d, (rank + 1) * gk * G * d
    out = {"x": inp["x"], "W_q": inp["W_q"][q0:q1], "W_k": inp["W_k"][k0:k1], "W_v": inp["W_v"][k0:k1],
           "W_o": inp["W_o"][:, q0:q1], "convq_seq": inp["convq_seq"][q0:q1], "convk_seq": inp["convk_seq"][k0:k1],
           "convq_chan": inp["convq_chan"][rank * gk * G:(rank + 1) * gk * G],
           "convk_chan": inp["convk_chan"][rank * gk:(rank + 1) * gk]}
    return out, gk * G, gk, nkv * d // 2 - k0  # the whole block's shift boundary in this share's channels


def _split_worker(rank, world, port, q, sh):
    import numpy as np

    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = workloads.as_float64(workloads.make_inputs(sh))
        mine, nq_r, nkv_r, vfrom = _share(inp, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, rank, world)
        part = oracle.cca_block(mine, nq_r, nkv_r, sh.head_dim, value_shift_from=vfrom)
        y = torch.from_numpy(np.ascontiguousarray(part["y"]))
        dist.all_reduce(y, op=dist.ReduceOp.SUM)  # the split's one exchange
        q.put((rank, y.numpy(), part["k_cache"], part["v_cache"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("nq,nkv", [(4, 2), (8, 4), (2, 2)])
def test_kv_group_split_sums_to_the_block(nq, nkv):
    import numpy as np

    import oracle
    d = 16
    sh = workloads.BlockShape("split", 2, 37, 2 * nq * d, nq, nkv, d, 4, "f32", 17)
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q, sh)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=180) for _ in range(world)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    full = oracle.cca_block(workloads.as_float64(workloads.make_inputs(sh)), nq, nkv, d)
    for rank, y, kc, vc in res:
        np.testing.assert_allclose(y, full["y"], rtol=1e-11, atol=1e-12)
        gk = nkv // world
        np.testing.assert_allclose(kc, full["k_cache"][:, :, rank * gk:(rank + 1) * gk], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(vc, full["v_cache"][:, :, rank * gk:(rank + 1) * gk], rtol=1e-12, atol=1e-13)
