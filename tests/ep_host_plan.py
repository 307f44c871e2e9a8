"""Host restatement of the expert-parallel plan (imported by tests only): which
requests each rank has accepted under token-order acceptance over the whole
routing group, how many rows go to each rank, and the regrouping of rows
received source-major into the owner's expert-major order.  The CPU protocol
test runs on it, and the GPU tests check the library's plan (moe_ep_plan)
against it."""
import numpy as np


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


def dest_base(acc: np.ndarray, rank: int, n_ranks: int) -> np.ndarray:
    """For each expert e, where rank `rank`'s first accepted row of e lands in
    the owner's expert-major buffer: rows of the owner's earlier experts plus
    the rows of e from earlier ranks."""
    R = n_ranks
    E = acc.shape[1]
    El = E // R
    tot = acc.sum(axis=0)
    out = np.zeros(E, np.int64)
    for e in range(E):
        owner0 = (e // El) * El
        out[e] = tot[owner0:e].sum() + acc[:rank, e].sum()
    return out
