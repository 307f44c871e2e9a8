"""The sharded routing group on CPU ranks (world size 2, gloo): the exchange of
per-rank request counts and the group-wide token-order acceptance give, on
every rank, exactly the single-batch routing records and outputs.

The per-rank computation here is the oracle's (there is no GPU); the exchange
and the rank offsets are the product's (sparse_mixture_experts_25_b200.sharded).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import seeded_inputs as si
from sparse_mixture_experts_25_b200 import sharded


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = si.WORKLOADS["qwen3_skew_bf16"].scaled("sharded", N=600, d=128, d_f=64, E=16, k=4)
        inp = si.inputs(w)
        lo, hi = sharded.shard_range(w.N, rank, world)
        x = inp["x"][lo:hi]
        r = oracle.route(x, inp["W_r"], k=w.k, norm=w.norm, b_r=inp["b_r"])
        ids = r["ids"]
        counts = torch.from_numpy(np.bincount(ids[ids >= 0], minlength=w.E).astype(np.int32))
        counts_all = sharded.exchange_counts(counts)
        base = sharded.rank_bases(counts_all, rank).numpy()
        C = oracle.capacity(w.c, w.N, w.k, w.E)        # the group's capacity
        d = oracle.dispatch_ranked(ids, E=w.E, C=C, base=base)
        Y = oracle.forward_rows(x, ids, r["w"], d["slot"], np.arange(hi - lo), inp["W_g"], inp["W_u"],
                                inp["W_d"])
        out_q.put((rank, lo, hi, ids, d["slot"], Y, counts_all.numpy()))
    finally:
        dist.destroy_process_group()


def test_sharded_group_equals_single_batch():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort(key=lambda t: t[0])
    # single-batch reference
    w = si.WORKLOADS["qwen3_skew_bf16"].scaled("sharded", N=600, d=128, d_f=64, E=16, k=4)
    inp = si.inputs(w)
    C = oracle.capacity(w.c, w.N, w.k, w.E)
    full = oracle.forward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], k=w.k, norm=w.norm,
                          c=w.c, b_r=inp["b_r"])
    assert full["stats"]["rejected"] > 0              # capacity binds across the shards
    ids = np.concatenate([t[3] for t in results])
    slot = np.concatenate([t[4] for t in results])
    Y = np.concatenate([t[5] for t in results])
    np.testing.assert_array_equal(ids, full["ids"])
    np.testing.assert_array_equal(slot, full["slot"])
    np.testing.assert_allclose(Y, full["Y"], rtol=1e-12, atol=1e-12)
    # both ranks saw the same gathered table, whose rows are the shards' counts
    np.testing.assert_array_equal(results[0][6], results[1][6])
    assert results[0][6].sum() == w.N * w.k


def test_rank_bases_and_ranges():
    counts_all = torch.tensor([[3, 0, 2], [1, 4, 0], [2, 2, 2]], dtype=torch.int32)
    assert sharded.rank_bases(counts_all, 0).tolist() == [0, 0, 0]
    assert sharded.rank_bases(counts_all, 2).tolist() == [4, 4, 2]
    assert [sharded.shard_range(10, r, 3) for r in range(3)] == [(0, 4), (4, 8), (8, 10)]


def _max_worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import bench
        out_q.put((rank, bench.max_over_ranks(1.5 + rank, device="cpu")))
    finally:
        dist.destroy_process_group()


def test_bench_time_is_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_max_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 2.5), (1, 2.5)]
