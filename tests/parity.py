"""Helpers for the GPU-vs-oracle parity tests (imported by tests only).

Comparison rules (stated once, used by every parity test):
  * routing ids are compared exactly for every token whose oracle score
    margin g_(k) - g_(k+1) is >= 1e-5 (and, under WLR, whose every pruning
    test has |ratio - theta| >= 1e-5); the others are near-ties: counted,
    reported and excluded from id equality;
  * dispatch is checked bit-exactly by running the oracle's dispatch on the
    GPU's own ids (one flipped near-tie would shift later slots otherwise);
  * weights: |a_gpu - a_oracle| <= 3e-5 (1 + |a|): the GPU accumulates router
    scores in fp32 over d products (two-level, 64-wide chunks), an error of
    order sqrt(d) 2^-24 |x||w| (~1e-6 .. 1e-5 at d = 4096..7168), and a
    softmax weight moves by at most about twice the largest score error;
  * outputs: max|Y_gpu - Y_ref| / max|Y_ref| <= 1e-4 (fp32 layers) or 2e-2
    (bf16 layers, fp32 accumulation), with Y_ref the oracle's output
    computed from the GPU's routing records, both over all compared rows
    (normwise) and row by row (each row's largest error over that row's
    largest reference entry), so one wrong row among many larger ones
    cannot hide; rows whose reference is zero (every path dropped, no
    shared expert) must be exactly zero.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import seeded_inputs as si

TOL = {si.DT_F32: 1e-4, si.DT_BF16: 2e-2}
NEAR = 1e-5


def torch_mod():
    import torch
    return torch


def to_dev(a):
    torch = torch_mod()
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def params_of(w: si.Workload):
    import sparse_mixture_experts_25_b200 as moe
    return moe.params(w.N, w.d, w.d_f, w.E, w.k, c=w.c, norm=w.norm, theta=w.theta,
                      dtype=w.dtype, d_f_shared=w.d_f_shared, reject_policy=w.reject_policy,
                      accept_order=w.accept_order, reroute_depth=w.reroute_depth)


def gpu_forward(w: si.Workload, inp: dict, dev: dict | None = None):
    """moe_forward through the C ABI; returns Y, routing records (host) and stats."""
    import sparse_mixture_experts_25_b200 as moe
    torch = torch_mod()
    p = params_of(w)
    if dev is None:
        dev = {k: to_dev(v) for k, v in inp.items()}
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    Y = torch.full((w.N, w.d), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_forward(p, dev["x"], dev["W_r"], dev.get("b_r"), dev.get("lat"), dev["W_g"], dev["W_u"],
                    dev["W_d"], dev.get("Ws_g"), dev.get("Ws_u"), dev.get("Ws_d"), Y, ws)
    status, stats = moe.moe_get_stats(p, ws)
    views = moe.workspace_views(p, ws)
    rec = {k: v.cpu().numpy() for k, v in views.items()}
    return {"Y": Y.cpu().numpy().astype(np.float64), "rec": rec, "stats": stats, "status": status,
            "ws": ws, "p": p, "dev": dev}


def check_routing(w: si.Workload, inp: dict, rec: dict):
    """Oracle routing on the same inputs; returns (oracle route dict, near-tie mask)."""
    r = oracle.route(inp["x"], inp["W_r"], k=w.k, norm=w.norm, theta=w.theta, b_r=inp.get("b_r"),
                     lat=inp.get("lat"))
    near = (r["margin"] < NEAR) | (r["wlr_gap"] < NEAR)
    ok = ~near & ~r["invalid"]
    assert (rec["ids"][ok] == r["ids"][ok]).all(), "routing ids differ on tokens that are not near-ties"
    same = ok[:, None] & (rec["ids"] == r["ids"])
    np.testing.assert_allclose(rec["w"][same], r["w"][same], rtol=3e-5, atol=3e-5)
    assert (rec["ids"][r["invalid"]] == -1).all()
    # margin reported by the GPU (fp32) agrees with the oracle's (double)
    fin = ok & np.isfinite(r["margin"])
    np.testing.assert_allclose(rec["margin"][fin], r["margin"][fin], rtol=1e-4, atol=2e-5)
    return r, near


def check_candidates(w: si.Workload, r: dict, rec: dict):
    """Rerouting candidates (ranks k .. k+X-1) against the oracle's, on the
    tokens whose scores around those ranks are not near-ties (every gap
    between consecutive ranks k-1 .. k+X at least 1e-5); weights within the
    routing-weight bound.  Returns the mask of compared tokens."""
    X = w.reroute_depth
    cand, cw = oracle.reroute_candidates(r["logits"], r["ids"], r["invalid"], w.k, X, w.norm)
    g = -np.sort(-r["logits"], axis=1)
    hi = min(w.E - 1, w.k + X)
    gaps = g[:, w.k - 1:hi] - g[:, w.k:hi + 1]
    clear = ~r["invalid"] & (gaps.min(axis=1) >= NEAR if gaps.shape[1] else True) & (r["margin"] >= NEAR)
    np.testing.assert_array_equal(rec["cand"][clear], cand[clear])
    np.testing.assert_allclose(rec["cand_w"][clear], cw[clear], rtol=3e-5, atol=3e-5)
    assert (rec["cand"][r["invalid"]] == -1).all()
    return clear


def check_dispatch_reroute(w: si.Workload, rec: dict, stats: dict):
    """Rerouting dispatch: the oracle's rounds on the GPU's own ids and
    candidates; first-choice slots, rerouted experts and slots, rows per
    expert, offsets, row records and statistics bit for bit."""
    C = oracle.capacity(w.c, w.N, w.k, w.E)
    d = oracle.dispatch_reroute(rec["ids"], rec["cand"], E=w.E, C=C)
    np.testing.assert_array_equal(rec["slot"], d["slot"])
    np.testing.assert_array_equal(rec["rr_e"], d["rr_e"])
    np.testing.assert_array_equal(rec["rr_slot"], d["rr_slot"])
    np.testing.assert_array_equal(rec["L"], d["L"])
    np.testing.assert_array_equal(rec["acc"], d["acc"])
    offs = np.concatenate([[0], np.cumsum(d["acc"])])
    np.testing.assert_array_equal(rec["offsets"], offs)
    ids2, w2, slot2 = oracle.served_records(rec["ids"], rec["w"].astype(np.float64), d["slot"], d["rr_e"],
                                            d["rr_slot"], d["rr_q"], rec["cand_w"].astype(np.float64))
    t_idx, j_idx = np.nonzero(slot2 >= 0)
    pos = offs[ids2[t_idx, j_idx]] + slot2[t_idx, j_idx]
    assert pos.size == offs[-1] and np.unique(pos).size == pos.size
    np.testing.assert_array_equal(rec["slot_token"][pos], t_idx)
    np.testing.assert_array_equal(rec["slot_w"][pos], w2[t_idx, j_idx].astype(np.float32))
    s = d["stats"]
    for key in ("requested", "accepted", "rejected", "O", "tokens_affected", "tokens_skipped", "L_max",
                "rerouted"):
        assert stats[key] == s[key], (key, stats[key], s[key])
    assert stats["C"] == C
    return d


def check_dispatch(w: si.Workload, rec: dict, stats: dict):
    """Oracle dispatch on the GPU's own ids (and, for acceptance by weight, on
    its own fp32 weights, so both sides order the requests by the same
    numbers): slots, loads, offsets, records and statistics must match bit
    for bit."""
    if w.reject_policy == 2:
        return check_dispatch_reroute(w, rec, stats)
    C = oracle.capacity(w.c, w.N, w.k, w.E)
    if w.accept_order == 1:
        d = oracle.dispatch_priority(rec["ids"], rec["w"].astype(np.float64), E=w.E, C=C)
    else:
        d = oracle.dispatch(rec["ids"], E=w.E, C=C)
    np.testing.assert_array_equal(rec["slot"], d["slot"])
    np.testing.assert_array_equal(rec["L"], d["L"])
    np.testing.assert_array_equal(rec["acc"], d["acc"])
    offs = np.concatenate([[0], np.cumsum(d["acc"])])
    np.testing.assert_array_equal(rec["offsets"], offs)
    # every accepted record sits at offsets[e] + slot with its token and weight
    t_idx, j_idx = np.nonzero(d["slot"] >= 0)
    pos = offs[rec["ids"][t_idx, j_idx]] + d["slot"][t_idx, j_idx]
    np.testing.assert_array_equal(rec["slot_token"][pos], t_idx)
    wc = oracle.reject_weights(rec["ids"], rec["w"].astype(np.float64), rec["slot"], w.reject_policy)
    if w.reject_policy == 0:
        np.testing.assert_array_equal(rec["slot_w"][pos], rec["w"][t_idx, j_idx])
    else:
        np.testing.assert_allclose(rec["slot_w"][pos], wc[t_idx, j_idx], rtol=1e-6, atol=1e-7)
    s = d["stats"]
    for key in ("requested", "accepted", "rejected", "O", "tokens_affected", "tokens_skipped", "L_max"):
        assert stats[key] == s[key], (key, stats[key], s[key])
    assert stats["C"] == C
    # tile padding of the routed GEMMs: each expert's accepted rows rounded up
    # to the row tile (64 rows for fp32 layers; 128, or 256 on CTA pairs when
    # experts average >= 768 rows, for bf16 layers).  On CTA pairs a tail of
    # at most 128 rows past the last 256-row boundary runs as one tile of its
    # rows rounded up to 32.
    pair = w.dtype != si.DT_F32 and w.N * w.k >= 768 * w.E
    bm = 64 if w.dtype == si.DT_F32 else (256 if pair else 128)

    def padded_rows(a):
        tail = a % 256 if pair and a % 256 <= 128 else 0
        rows = -(-(a - tail) // bm) * bm + -(-tail // 32) * 32
        # single-CTA tensor-core tiles: a last tile of at most 64 rows is an M=64 MMA
        if bm == 128 and 0 < a % 128 <= 64:
            rows -= 64
        return rows

    padded = int(sum(padded_rows(int(a)) for a in d["acc"]))
    assert stats["padded_rows"] == padded
    assert stats["padding_ratio"] == pytest.approx(padded / s["accepted"] if s["accepted"] else 0.0)
    if w.N:
        assert abs(stats["rho_max"] - oracle.rho_max(d["L"], w.N, w.k, w.E)) < 1e-12
        for q, key in ((50, "L_p50"), (90, "L_p90"), (99, "L_p99")):
            assert stats[key] == oracle.load_percentile(d["L"], q)
    return d


def rel_err(Y, Yref) -> float:
    den = float(np.max(np.abs(Yref))) if Yref.size else 0.0
    return float(np.max(np.abs(Y - Yref))) / (den if den > 0 else 1.0)


def row_rel_err(Y, Yref) -> float:
    """Largest per-row error: max over rows of max|Y_i - Yref_i| / max|Yref_i|.
    A row whose reference is exactly zero must be exactly zero (its error is
    infinite otherwise)."""
    if Yref.size == 0:
        return 0.0
    den = np.max(np.abs(Yref), axis=1)
    num = np.max(np.abs(Y - Yref), axis=1)
    zero = den == 0
    if (num[zero] != 0).any():
        return float("inf")
    if zero.all():
        return 0.0
    return float(np.max(num[~zero] / den[~zero]))


def assert_rows_close(Y, Yref, tol) -> tuple:
    """Normwise and per-row max-abs-rel bounds; returns both errors."""
    err = rel_err(Y, Yref)
    row = row_rel_err(Y, Yref)
    assert err <= tol, f"max-abs-rel error {err:.3e} above {tol:.0e}"
    assert row <= tol, f"largest per-row max-abs-rel error {row:.3e} above {tol:.0e}"
    return err, row


def last_tile_tokens(rec: dict, tile: int = 256) -> np.ndarray:
    """Tokens of every accepted row in each expert's last `tile`-row block of
    its buffer (the block that ends mid-tile when the expert's row count is
    not a multiple of the tile; the full last block otherwise).  With tile =
    256 this covers the last row tile of every tile height the GEMMs use
    (128, 256 rows, or token tiles of up to 256)."""
    offs = np.asarray(rec["offsets"], np.int64)
    st = np.asarray(rec["slot_token"])
    toks = []
    for e in range(offs.size - 1):
        lo, hi = int(offs[e]), int(offs[e + 1])
        if hi > lo:
            start = lo + ((hi - lo - 1) // tile) * tile
            toks.append(st[start:hi])
    if not toks:
        return np.zeros(0, np.int64)
    return np.unique(np.concatenate(toks).astype(np.int64))


def check_rows(w: si.Workload, inp: dict, rec: dict, Y: np.ndarray, tokens=None):
    """Y rows against the oracle evaluated on the GPU's routing records;
    returns (normwise error, largest per-row error)."""
    if tokens is None:
        tokens = np.arange(w.N)
    Ws = (inp.get("Ws_g"), inp.get("Ws_u"), inp.get("Ws_d")) if w.d_f_shared else None
    if w.reject_policy == 2:
        # every served path: first choices and rerouted ones, from the GPU's records
        C = oracle.capacity(w.c, w.N, w.k, w.E)
        d = oracle.dispatch_reroute(rec["ids"], rec["cand"], E=w.E, C=C)
        ids2, wc, slot2 = oracle.served_records(rec["ids"], rec["w"].astype(np.float64), d["slot"], d["rr_e"],
                                                d["rr_slot"], d["rr_q"], rec["cand_w"].astype(np.float64))
    else:
        ids2, slot2 = rec["ids"], rec["slot"]
        wc = oracle.reject_weights(rec["ids"], rec["w"].astype(np.float64), rec["slot"], w.reject_policy)
    ref = oracle.forward_rows(inp["x"], ids2, wc, slot2, tokens,
                              inp["W_g"], inp["W_u"], inp["W_d"], Ws=Ws)
    err, row = assert_rows_close(Y[tokens], ref, TOL[w.dtype])
    dropped = [i for i, t in enumerate(tokens) if not w.d_f_shared and (slot2[t] < 0).all()]
    for i in dropped:
        assert (Y[tokens[i]] == 0).all()
    return err, row
