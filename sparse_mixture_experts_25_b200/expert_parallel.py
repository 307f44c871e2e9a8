"""Expert parallelism for the MoE layer ("LLM from scratch" ch. 36.7: expert
parameters placed on different devices; after routing, token rows go to the
device of their expert and the expert outputs come back).

Rank r of R owns experts [r E/R, (r+1) E/R) and holds a contiguous shard of the
routing group's tokens (rank order = token order).  One layer step:

  1. route this rank's tokens and count requests per expert (moe_forward_begin);
  2. all-gather the counts: every rank then knows, for every rank and expert,
     how many requests are accepted (capacity over the whole group, token order);
  3. accept this rank's requests and gather their rows grouped by expert
     (moe_dispatch_ranked): the rows bound for rank r' form one contiguous
     block of x_perm, since r' owns a contiguous range of experts;
  4. all-to-all of those blocks; the received rows (source-major) are regrouped
     expert-major (moe_gather_rows);
  5. the owned experts on their rows (moe_expert_ffn);
  6. the outputs back to source-major order and all-to-all back: each rank gets
     the outputs of its own rows, in its x_perm order;
  7. the weighted combine into token order (moe_combine); the shared expert, if
     any, is replicated on every rank and applied to the rank's own tokens.

The result equals the single-GPU layer on the concatenated batch.  The
exchanges are torch.distributed collectives (NCCL between GPUs); every step of
the arithmetic runs in libmoe's kernels.  The per-destination row counts of
the all-to-alls are taken from the exchanged counts on the host (one small
device-to-host copy per step).
"""
from __future__ import annotations

from typing import Optional

import numpy as np

import sparse_mixture_experts_25_b200 as moe


def accepted_counts(counts_all, C: int) -> np.ndarray:
    """acc[s, e]: requests of rank s for expert e that the group accepts, with
    requests taken in group token order (earlier ranks first) up to C per
    expert."""
    L = np.asarray(counts_all, np.int64)
    base = np.cumsum(L, axis=0) - L
    return np.clip(C - base, 0, L)


def send_rows(acc: np.ndarray, n_ranks: int) -> np.ndarray:
    """rows[s, r]: rows rank s sends to rank r (its accepted requests for the
    experts rank r owns)."""
    R = n_ranks
    El = acc.shape[1] // R
    return acc.reshape(R, R, El).sum(axis=2)


def regroup(acc: np.ndarray, rank: int, n_ranks: int):
    """On `rank`, received rows arrive source-major (source s, then the owned
    experts in order).  Returns (index, offsets): received row index[i] is the
    i-th row in expert-major order (owned expert j, then source s), and
    offsets[j] .. offsets[j+1]-1 are expert j's rows in that order."""
    R = n_ranks
    El = acc.shape[1] // R
    seg = acc[:, rank * El:(rank + 1) * El]                      # [source, owned expert]
    src_start = np.concatenate([[0], np.cumsum(seg.sum(axis=1))[:-1]])
    within = np.cumsum(seg, axis=1) - seg
    parts, offsets = [], [0]
    for j in range(El):
        for s in range(R):
            st = int(src_start[s] + within[s, j])
            parts.append(np.arange(st, st + int(seg[s, j]), dtype=np.int64))
        offsets.append(offsets[-1] + int(seg[:, j].sum()))
    index = np.concatenate(parts) if parts else np.zeros(0, np.int64)
    return index.astype(np.int32), np.asarray(offsets, np.int32)


class ExpertParallelLayer:
    """One rank's share of an expert-parallel MoE layer.

    p: this rank's layer parameters (p.N = its tokens, full E_r, capacity
    factor of the group).  W_g, W_u, W_d: the owned experts' weights
    [E_r / R, ...].  W_r (and b_r, lat) replicated; shared = (Ws_g, Ws_u,
    Ws_d) replicated or None.  Token-order acceptance only."""

    def __init__(self, p: "moe.Params", rank: int, n_ranks: int, N_group: int, W_r, W_g, W_u, W_d,
                 b_r=None, lat=None, shared=None, device="cuda"):
        import torch
        if p.E_r % n_ranks:
            raise ValueError("the experts must split evenly over the ranks")
        self.torch = torch
        self.p, self.rank, self.R, self.N_group = p, rank, n_ranks, N_group
        self.El = p.E_r // n_ranks
        self.W_r, self.b_r, self.lat = W_r, b_r, lat
        self.W = (W_g, W_u, W_d)
        self.C = moe.moe_capacity(moe.params(N_group, p.d, p.d_f, p.E_r, p.k, c=p.c, norm=p.norm, theta=p.theta,
                                             dtype=p.dtype, d_f_shared=p.d_f_shared))
        dt = torch.bfloat16 if p.dtype == moe.MOE_BF16 else torch.float32
        self.ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device=device)
        self.counts = torch.empty(p.E_r, dtype=torch.int32, device=device)
        # the owned experts' rows: at most C per expert
        rows = max(1, self.El * self.C)
        self.p_loc = moe.params(rows, p.d, p.d_f, self.El, 1, dtype=p.dtype)
        self.ws_loc = torch.empty(moe.moe_workspace_size(self.p_loc), dtype=torch.uint8, device=device)
        self.x_loc = torch.empty(rows, p.d, dtype=dt, device=device)
        self.h_loc = torch.empty(rows, p.d, dtype=torch.float32, device=device)
        self.h_send = torch.empty(rows, p.d, dtype=torch.float32, device=device)
        self.h_back = torch.empty(max(1, p.N * p.k), p.d, dtype=torch.float32, device=device)
        self.shared = shared
        if shared is not None:
            Ws_g, Ws_u, Ws_d = shared
            self.p_sh = moe.params(p.N, p.d, Ws_g.shape[0], 1, 1, dtype=p.dtype)
            self.ws_sh = torch.empty(moe.moe_workspace_size(self.p_sh), dtype=torch.uint8, device=device)
            self.sh_w = (Ws_g.unsqueeze(0), Ws_u.unsqueeze(0), Ws_d.unsqueeze(0))
            self.h_sh = torch.empty(max(1, p.N), p.d, dtype=torch.float32, device=device)
            self.sh_offsets = torch.tensor([0, p.N], dtype=torch.int32, device=device)
            self.sh_token = torch.arange(p.N, dtype=torch.int32, device=device)
            self.sh_w1 = torch.ones(p.N, dtype=torch.float32, device=device)

    # -- phases ---------------------------------------------------------------
    def route(self, x, stream=None):
        """Step 1: routing and this rank's per-expert request counts."""
        moe.moe_forward_begin(self.p, x, self.W_r, self.b_r, self.lat, self.counts, self.ws, stream)
        return self.counts

    def dispatch(self, x, counts_all, counts_host, stream=None):
        """Step 3: returns (send buffer [rows, d], rows per destination rank)."""
        moe.moe_dispatch_ranked(self.p, counts_all, self.rank, self.R, self.N_group, self.C, x, self.ws, stream)
        self.acc = accepted_counts(counts_host, self.C)
        self.rows_to = send_rows(self.acc, self.R)
        n = int(self.rows_to[self.rank].sum())
        return moe.workspace_x_perm(self.p, self.ws)[:n], [int(v) for v in self.rows_to[self.rank]]

    def experts(self, recv, stream=None):
        """Steps 4-6a: received rows (source-major) -> owned experts ->
        outputs in source-major order; returns (outputs, rows per source)."""
        torch = self.torch
        index, offsets = regroup(self.acc, self.rank, self.R)
        n = int(index.size)
        dev = recv.device
        if n:
            inverse = np.empty(n, np.int32)
            inverse[index] = np.arange(n, dtype=np.int32)
            idx = torch.from_numpy(index).to(dev)
            inv = torch.from_numpy(inverse).to(dev)
            moe.moe_gather_rows(recv, idx, self.x_loc[:n], stream)
            off = torch.from_numpy(offsets).to(dev)
            moe.moe_expert_ffn(self.p_loc, self.x_loc, off, *self.W, self.h_loc, self.ws_loc, stream)
            moe.moe_gather_rows(self.h_loc, inv, self.h_send[:n], stream)
        return self.h_send[:n], [int(v) for v in self.rows_to[:, self.rank]]

    def combine(self, h_back, x, Y, stream=None):
        """Step 7: Y = weighted combine of this rank's returned outputs (+ the
        shared expert on its tokens)."""
        torch = self.torch
        views = moe.workspace_views(self.p, self.ws)
        if stream is None:
            Y.zero_()
        else:
            with torch.cuda.stream(stream if not isinstance(stream, int) else torch.cuda.ExternalStream(stream)):
                Y.zero_()
        n = int(h_back.shape[0])
        if n:
            moe.moe_combine(self.p, h_back, views["offsets"], views["slot_token"], views["slot_w"], Y, stream)
        if self.shared is not None and self.p.N:
            moe.moe_expert_ffn(self.p_sh, x, self.sh_offsets, *self.sh_w, self.h_sh, self.ws_sh, stream)
            moe.moe_combine(self.p_sh, self.h_sh, self.sh_offsets, self.sh_token, self.sh_w1, Y, stream)

    # -- one step with torch.distributed collectives ---------------------------
    def forward(self, x, Y, group=None, stream=None):
        torch = self.torch
        import torch.distributed as dist
        st = torch.cuda.current_stream(x.device) if stream is None else stream
        with torch.cuda.stream(st):
            counts = self.route(x, st)
            parts = [torch.empty_like(counts) for _ in range(self.R)]
            dist.all_gather(parts, counts, group=group)
            counts_all = torch.stack(parts)
            counts_host = counts_all.cpu().numpy()
            send, split_out = self.dispatch(x, counts_all, counts_host, st)
            split_in = [int(v) for v in send_rows(accepted_counts(counts_host, self.C), self.R)[:, self.rank]]
            recv = torch.empty(sum(split_in), self.p.d, dtype=send.dtype, device=x.device)
            dist.all_to_all_single(recv, send.contiguous(), split_in, split_out, group=group)
            out, back_split_out = self.experts(recv, st)
            back = self.h_back[:sum(split_out)]
            dist.all_to_all_single(back, out.contiguous(), split_out, back_split_out, group=group)
            self.combine(back, x, Y, st)
        return Y


def emulate(layers, xs, Ys, stream=None):
    """All ranks of one expert-parallel step in one process (one GPU): the
    collectives become copies in rank order.  For tests and single-GPU use."""
    import torch
    R = len(layers)
    counts = [L.route(x, stream) for L, x in zip(layers, xs)]
    counts_all = torch.stack(counts)
    counts_host = counts_all.cpu().numpy()
    sends = [L.dispatch(x, counts_all, counts_host, stream) for L, x in zip(layers, xs)]
    outs = []
    for r, L in enumerate(layers):
        blocks = []
        for s in range(R):
            buf, split = sends[s]
            lo = sum(split[:r])
            blocks.append(buf[lo:lo + split[r]])
        recv = torch.cat(blocks) if blocks else sends[0][0][:0]
        outs.append(L.experts(recv, stream))
    for s, (L, x, Y) in enumerate(zip(layers, xs, Ys)):
        blocks = []
        for r in range(R):
            buf, split = outs[r]
            lo = sum(split[:s])
            blocks.append(buf[lo:lo + split[s]])
        L.combine(torch.cat(blocks), x, Y, stream)
    return Ys
