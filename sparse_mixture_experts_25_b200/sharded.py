"""Forward pass over a routing group whose tokens are sharded across ranks.

Data parallel: every rank holds the same weights and a shard of the group's
tokens, ranks in token order (rank 0's tokens first).  Capacity competition
is defined over the whole routing group, so the ranks exchange one table, the
per-expert request counts of every rank (E_r int32 each), between the two
library calls moe_forward_begin and moe_forward_end.  The result on every
rank is exactly what one GPU computes for the concatenated batch.

The exchange is a torch.distributed all-gather (NCCL between GPUs); all
arithmetic of the layer runs in libmoe's kernels.
"""
from __future__ import annotations

from typing import Optional

import sparse_mixture_experts_25_b200 as moe


def exchange_counts(counts, group=None):
    """All-gather of the per-rank request counts: [n_ranks, E_r], rank order."""
    import torch
    import torch.distributed as dist
    n = dist.get_world_size(group)
    parts = [torch.empty_like(counts) for _ in range(n)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts)


def rank_bases(counts_all, rank: int):
    """Requests for each expert made by the tokens of earlier ranks: the
    offset of this rank's requests in the group's token order."""
    if rank == 0:
        return counts_all[0] * 0
    return counts_all[:rank].sum(dim=0)


def forward_sharded(p_local: "moe.Params", N_group: int, C: int, x, W_r, b_r, lat, W_g, W_u, W_d,
                    Ws_g, Ws_u, Ws_d, Y, ws, group=None, counts=None, stream=None):
    """One layer forward for this rank's shard (p_local.N tokens of a group of
    N_group tokens; C = the group's capacity).  Y [p_local.N, d] is written."""
    import torch
    import torch.distributed as dist
    if counts is None:
        counts = torch.empty(p_local.E_r, dtype=torch.int32, device=x.device)
    moe.moe_forward_begin(p_local, x, W_r, b_r, lat, counts, ws, stream)
    # the exchange runs on the layer's stream, after the counts are written
    if stream is None:
        st = torch.cuda.current_stream(x.device)
    elif isinstance(stream, int):
        st = torch.cuda.ExternalStream(stream, device=x.device)
    else:
        st = stream
    with torch.cuda.stream(st):
        counts_all = exchange_counts(counts, group)
    moe.moe_forward_end(p_local, counts_all, dist.get_rank(group), dist.get_world_size(group),
                        N_group, C, x, W_g, W_u, W_d, Ws_g, Ws_u, Ws_d, Y, ws, stream)
    return counts_all


def shard_range(N_group: int, rank: int, n_ranks: int, per_rank: Optional[int] = None):
    """Token range [lo, hi) of a rank: contiguous blocks in rank order."""
    if per_rank is None:
        per_rank = (N_group + n_ranks - 1) // n_ranks
    lo = min(N_group, rank * per_rank)
    return lo, min(N_group, lo + per_rank)
