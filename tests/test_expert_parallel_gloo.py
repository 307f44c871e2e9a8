"""The expert-parallel exchange protocol on CPU ranks (world size 2, gloo):
counts all-gathered, rows sent to the rank that owns their expert, regrouped
expert-major, processed, sent back and combined.  The per-rank arithmetic is
the oracle's (no GPU); the plan, split sizes and regrouping are the product's
(sparse_mixture_experts_25_b200.expert_parallel), and the collectives are real.
The result equals the oracle's single-batch forward."""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import seeded_inputs as si
from tests import ep_host_plan as ep
from sparse_mixture_experts_25_b200 import sharded

CASE = si.WORKLOADS["qwen3_skew_bf16"].scaled("ep_gloo", N=400, d=64, d_f=32, E=8, k=2, dtype=si.DT_F32)


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = CASE
        inp = si.inputs(w)
        lo, hi = sharded.shard_range(w.N, rank, world)
        x = inp["x"][lo:hi]
        r = oracle.route(x, inp["W_r"], k=w.k, norm=w.norm, b_r=inp["b_r"])
        ids = r["ids"]
        counts = torch.from_numpy(np.bincount(ids[ids >= 0], minlength=w.E).astype(np.int64))
        parts = [torch.empty_like(counts) for _ in range(world)]
        dist.all_gather(parts, counts)
        counts_all = torch.stack(parts).numpy()
        C = oracle.capacity(w.c, w.N, w.k, w.E)
        base = counts_all[:rank].sum(axis=0)
        d = oracle.dispatch_ranked(ids, E=w.E, C=C, base=base)
        acc = ep.accepted_counts(counts_all, C)
        np.testing.assert_array_equal(acc[rank], d["acc"])
        # x_perm: accepted rows grouped by expert, token order inside an expert
        rows = [(e, t) for e in range(w.E) for t in range(hi - lo) for j in range(w.k)
                if ids[t, j] == e and d["slot"][t, j] >= 0]
        xp = np.stack([x[t].astype(np.float64) for _, t in rows]) if rows else np.zeros((0, w.d))
        rows_to = ep.send_rows(acc, world)
        send = torch.from_numpy(xp)
        recv = torch.empty(int(rows_to[:, rank].sum()), w.d, dtype=torch.float64)
        dist.all_to_all_single(recv, send, [int(v) for v in rows_to[:, rank]], [int(v) for v in rows_to[rank]])
        index, offsets = ep.regroup(acc, rank, world)
        xl = recv.numpy()[index]
        El = w.E // world
        hl = np.zeros_like(xl)
        for j in range(El):
            e = rank * El + j
            blk = np.ascontiguousarray(xl[offsets[j]:offsets[j + 1]])
            if blk.size:
                hl[offsets[j]:offsets[j + 1]] = oracle_dense(blk, inp, e)
        inv = np.empty_like(index)
        inv[index] = np.arange(index.size)
        back_send = torch.from_numpy(hl[inv] if hl.size else hl)
        back = torch.empty(len(rows), w.d, dtype=torch.float64)
        dist.all_to_all_single(back, back_send, [int(v) for v in rows_to[rank]], [int(v) for v in rows_to[:, rank]])
        Y = np.zeros((hi - lo, w.d))
        pos = {}
        for i, (e, t) in enumerate(rows):
            pos[(t, e)] = i
        for t in range(hi - lo):
            for j in range(w.k):
                e = ids[t, j]
                if e >= 0 and d["slot"][t, j] >= 0:
                    Y[t] += r["w"][t, j] * back.numpy()[pos[(t, e)]]
        out_q.put((rank, Y))
    finally:
        dist.destroy_process_group()


def oracle_dense(rows, inp, e):
    out = np.empty_like(rows)
    lib = oracle._load()
    lib.oracle_swiglu_dense(rows.shape[1], inp["W_g"].shape[1], 0, 0, oracle._ptr(rows), rows.shape[0],
                            oracle._ptr(np.ascontiguousarray(inp["W_g"][e])),
                            oracle._ptr(np.ascontiguousarray(inp["W_u"][e])),
                            oracle._ptr(np.ascontiguousarray(inp["W_d"][e])), oracle._ptr(out))
    return out


def test_expert_parallel_protocol_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted([q.get(timeout=300) for _ in range(2)], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = CASE
    inp = si.inputs(w)
    full = oracle.forward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], k=w.k, norm=w.norm, c=w.c,
                          b_r=inp["b_r"])
    assert full["stats"]["rejected"] > 0          # capacity binds across the ranks
    Y = np.concatenate([g[1] for g in got])
    np.testing.assert_allclose(Y, full["Y"], rtol=1e-10, atol=1e-12)
