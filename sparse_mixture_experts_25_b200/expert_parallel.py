"""Expert parallelism for the MoE layer ("LLM from scratch" ch. 36.7: expert
parameters placed on different devices; after routing, token rows go to the
device of their expert and the expert outputs come back).

Rank r of R owns experts [r E/R, (r+1) E/R) and holds a contiguous shard of the
routing group's tokens (rank order = token order).  Every step starts the same
way:

  1. route this rank's tokens and count requests per expert (moe_forward_begin);
  2. all-gather the counts (the one exchange every rank needs before it knows
     which of its requests the group accepts: capacity over the whole group,
     token order);
  3. accept this rank's requests (moe_dispatch_ranked) and derive the plan of
     the step on the device (moe_ep_plan): where each accepted row lands in its
     owner's expert-major buffer, the owned experts' row offsets, the rows sent
     to and received from each rank.

Two ways to move the rows:

  * fused (forward_peer / emulate_peer): moe_ep_dispatch writes every accepted
    row straight into its owner's expert-major buffer (a peer GPU's memory over
    NVLink), the owners run their experts (moe_expert_ffn) in place, and
    moe_ep_combine reads each output row straight from its owner's buffer into
    the weighted combine.  Two barriers across the ranks order the phases.  No
    all-to-all, no regrouping, no host round trip.
  * collectives (forward / emulate): x_perm's expert blocks travel by NCCL
    all-to-all (torch.distributed) with the split sizes the plan kernel wrote
    (one small device-to-host copy), are regrouped expert-major with the plan's
    index (moe_gather_rows), and come back the same way before moe_combine.

The shared expert, if any, is replicated and applied on every rank to its own
tokens.  The result equals the single-GPU layer on the concatenated batch.
Every step of the arithmetic, including the plan, runs in libmoe's kernels.
"""
from __future__ import annotations

import sparse_mixture_experts_25_b200 as moe


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
        i32 = dict(dtype=torch.int32, device=device)
        self.ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device=device)
        self.counts = torch.empty(p.E_r, **i32)
        # the owned experts' rows: at most C per expert (expert-major)
        rows = max(1, self.El * self.C)
        self.p_loc = moe.params(rows, p.d, p.d_f, self.El, 1, dtype=p.dtype)
        self.ws_loc = torch.empty(moe.moe_workspace_size(self.p_loc), dtype=torch.uint8, device=device)
        self.x_loc = torch.empty(rows, p.d, dtype=dt, device=device)      # rows received (expert-major)
        self.h_loc = torch.empty(rows, p.d, dtype=torch.float32, device=device)  # their expert outputs
        self.h_send = torch.empty(rows, p.d, dtype=torch.float32, device=device)
        self.h_back = torch.empty(max(1, p.N * p.k), p.d, dtype=torch.float32, device=device)
        # the plan (written by moe_ep_plan)
        self.local_offsets = torch.empty(self.El + 1, **i32)
        self.splits = torch.empty(2 * n_ranks, **i32)        # send rows [R], then receive rows [R]
        self.regroup = torch.empty(rows, **i32)
        self.regroup_inv = torch.empty(rows, **i32)
        self.shared = shared
        if shared is not None:
            Ws_g, Ws_u, Ws_d = shared
            self.p_sh = moe.params(p.N, p.d, Ws_g.shape[0], 1, 1, dtype=p.dtype)
            self.ws_sh = torch.empty(moe.moe_workspace_size(self.p_sh), dtype=torch.uint8, device=device)
            self.sh_w = (Ws_g.unsqueeze(0), Ws_u.unsqueeze(0), Ws_d.unsqueeze(0))
            self.h_sh = torch.empty(max(1, p.N), p.d, dtype=torch.float32, device=device)
            self.sh_offsets = torch.tensor([0, p.N], **i32)
            self.sh_token = torch.arange(p.N, **i32)
            self.sh_w1 = torch.ones(p.N, dtype=torch.float32, device=device)

    # -- phases shared by both exchanges -----------------------------------------
    def route(self, x, stream=None):
        """Step 1: routing and this rank's per-expert request counts."""
        moe.moe_forward_begin(self.p, x, self.W_r, self.b_r, self.lat, self.counts, self.ws, stream)
        return self.counts

    def plan(self, x, counts_all, regroup: bool, stream=None):
        """Step 3: this rank's acceptance (rows gathered into x_perm when x is
        given) and the device plan of the step."""
        moe.moe_dispatch_ranked(self.p, counts_all, self.rank, self.R, self.N_group, self.C, x, self.ws, stream)
        moe.moe_ep_plan(self.p, counts_all, self.rank, self.R, self.C, self.local_offsets, self.splits[:self.R],
                        self.splits[self.R:], self.ws, regroup=self.regroup if regroup else None,
                        regroup_inv=self.regroup_inv if regroup else None, stream=stream)

    def owned_experts(self, stream=None):
        """The owned experts on the expert-major rows x_loc -> h_loc (their
        row counts are the plan's local offsets, on the device)."""
        moe.moe_expert_ffn(self.p_loc, self.x_loc, self.local_offsets, *self.W, self.h_loc, self.ws_loc, stream)

    def combine_shared(self, x, Y, stream=None):
        if self.shared is not None and self.p.N:
            moe.moe_expert_ffn(self.p_sh, x, self.sh_offsets, *self.sh_w, self.h_sh, self.ws_sh, stream)
            moe.moe_combine(self.p_sh, self.h_sh, self.sh_offsets, self.sh_token, self.sh_w1, Y, stream)

    def _zero(self, Y, stream):
        torch = self.torch
        if stream is None:
            Y.zero_()
        else:
            with torch.cuda.stream(stream if not isinstance(stream, int) else torch.cuda.ExternalStream(stream)):
                Y.zero_()

    # -- fused exchange: rows written to / read from the owners' buffers ---------
    def peer_dispatch(self, x, recv_table, stream=None):
        """This rank's accepted rows into their owners' expert-major buffers
        (recv_table: moe.pointer_table of every rank's x_loc)."""
        moe.moe_ep_dispatch(self.p, self.R, x, recv_table, self.ws, stream)

    def peer_combine(self, x, Y, out_table, stream=None):
        """Y = weighted outputs read from the owners' h_loc buffers (out_table:
        moe.pointer_table of every rank's h_loc), plus the shared expert."""
        self._zero(Y, stream)
        moe.moe_ep_combine(self.p, self.R, out_table, Y, self.ws, stream)
        self.combine_shared(x, Y, stream)

    def forward_peer(self, x, Y, recv_table, out_table, barrier, group=None, stream=None):
        """One step with the exchange fused into the dispatch and the combine.
        recv_table / out_table: device pointer tables of every rank's x_loc /
        h_loc (peer-accessible memory, e.g. torch symmetric memory);
        barrier(): orders every rank's previous kernels before any rank's next
        ones (e.g. a symmetric-memory barrier on the stream)."""
        torch = self.torch
        import torch.distributed as dist
        st = torch.cuda.current_stream(x.device) if stream is None else stream
        with torch.cuda.stream(st):
            counts = self.route(x, st)
            parts = [torch.empty_like(counts) for _ in range(self.R)]
            dist.all_gather(parts, counts, group=group)
            self.plan(None, torch.stack(parts), regroup=False, stream=st)
            self.peer_dispatch(x, recv_table, st)
            barrier()
            self.owned_experts(st)
            barrier()
            self.peer_combine(x, Y, out_table, st)
        return Y

    # -- collectives: NCCL all-to-all with the plan's split sizes ----------------
    def split_sizes(self):
        """(rows sent to each rank, rows received from each rank), as written
        by the plan kernel (one small device-to-host copy)."""
        s = self.splits.cpu().tolist()
        return s[:self.R], s[self.R:]

    def experts(self, recv, split_in, stream=None):
        """Received rows (source-major) -> expert-major -> owned experts ->
        outputs back in source-major order."""
        n = int(sum(split_in))
        if n:
            moe.moe_gather_rows(recv, self.regroup[:n], self.x_loc[:n], stream)
            self.owned_experts(stream)
            moe.moe_gather_rows(self.h_loc, self.regroup_inv[:n], self.h_send[:n], stream)
        return self.h_send[:n]

    def combine(self, h_back, x, Y, stream=None):
        """Y = weighted combine of this rank's returned outputs (+ the shared
        expert on its tokens)."""
        views = moe.workspace_views(self.p, self.ws)
        self._zero(Y, stream)
        if int(h_back.shape[0]):
            moe.moe_combine(self.p, h_back, views["offsets"], views["slot_token"], views["slot_w"], Y, stream)
        self.combine_shared(x, Y, stream)

    def forward(self, x, Y, group=None, stream=None):
        torch = self.torch
        import torch.distributed as dist
        st = torch.cuda.current_stream(x.device) if stream is None else stream
        with torch.cuda.stream(st):
            counts = self.route(x, st)
            parts = [torch.empty_like(counts) for _ in range(self.R)]
            dist.all_gather(parts, counts, group=group)
            self.plan(x, torch.stack(parts), regroup=True, stream=st)
            split_out, split_in = self.split_sizes()
            send = moe.workspace_x_perm(self.p, self.ws)[:sum(split_out)]
            recv = torch.empty(sum(split_in), self.p.d, dtype=send.dtype, device=x.device)
            dist.all_to_all_single(recv, send.contiguous(), split_in, split_out, group=group)
            out = self.experts(recv, split_in, st)
            back = self.h_back[:sum(split_out)]
            dist.all_to_all_single(back, out.contiguous(), split_out, split_in, group=group)
            self.combine(back, x, Y, st)
        return Y


def peer_buffers(layer: ExpertParallelLayer, group=None, timeout_ms: int = 10000):
    """Multi-GPU set-up of the fused exchange: the layer's expert-major buffers
    (x_loc for the rows received, h_loc for their outputs) are re-allocated in
    torch symmetric memory, every rank's addresses are exchanged, and a
    device-side barrier across the ranks (bounded by timeout_ms) orders the
    phases.  Returns (recv_table, out_table, barrier) for forward_peer.  The
    kernels reach the peers' buffers with plain loads and stores over NVLink.
    Needs one GPU per rank."""
    import torch
    import torch.distributed._symmetric_memory as symm_mem
    rows, d = layer.x_loc.shape
    dev = layer.x_loc.device
    layer.x_loc = symm_mem.empty(rows, d, dtype=layer.x_loc.dtype, device=dev)
    layer.h_loc = symm_mem.empty(rows, d, dtype=torch.float32, device=dev)
    hx = symm_mem.rendezvous(layer.x_loc, group if group is not None else torch.distributed.group.WORLD)
    hh = symm_mem.rendezvous(layer.h_loc, group if group is not None else torch.distributed.group.WORLD)
    recv_table = moe.pointer_table(list(hx.buffer_ptrs), device=dev)
    out_table = moe.pointer_table(list(hh.buffer_ptrs), device=dev)

    def barrier():
        hx.barrier(channel=0, timeout_ms=timeout_ms)

    return recv_table, out_table, barrier


def emulate(layers, xs, Ys, stream=None):
    """All ranks of one step of the collectives path in one process (one GPU):
    the collectives become copies in rank order.  For tests and single-GPU use."""
    import torch
    R = len(layers)
    counts_all = torch.stack([L.route(x, stream) for L, x in zip(layers, xs)])
    sends = []
    for L, x in zip(layers, xs):
        L.plan(x, counts_all, regroup=True, stream=stream)
        split_out, split_in = L.split_sizes()
        sends.append((moe.workspace_x_perm(L.p, L.ws)[:sum(split_out)], split_out, split_in))
    outs = []
    for r, L in enumerate(layers):
        blocks = []
        for s in range(R):
            buf, split, _ = sends[s]
            lo = sum(split[:r])
            blocks.append(buf[lo:lo + split[r]])
        outs.append((L.experts(torch.cat(blocks), sends[r][2], stream), sends[r][2]))
    for s, (L, x, Y) in enumerate(zip(layers, xs, Ys)):
        blocks = []
        for r in range(R):
            buf, split = outs[r]
            lo = sum(split[:s])
            blocks.append(buf[lo:lo + split[s]])
        L.combine(torch.cat(blocks), x, Y, stream)
    return Ys


def emulate_peer(layers, xs, Ys, stream=None):
    """All ranks of one step of the fused path in one process (one GPU): the
    owners' buffers are this GPU's memory and the phases run rank after rank
    (no rank waits on another).  For tests and single-GPU use."""
    import torch
    counts_all = torch.stack([L.route(x, stream) for L, x in zip(layers, xs)])
    recv_table = moe.pointer_table([L.x_loc for L in layers])
    out_table = moe.pointer_table([L.h_loc for L in layers])
    for L, x in zip(layers, xs):
        L.plan(None, counts_all, regroup=False, stream=stream)
    for L, x in zip(layers, xs):
        L.peer_dispatch(x, recv_table, stream)
    for L in layers:
        L.owned_experts(stream)
    for L, x, Y in zip(layers, xs, Ys):
        L.peer_combine(x, Y, out_table, stream)
    return Ys
