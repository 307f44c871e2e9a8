"""Pins of the oracle's rerouting overflow policy ("LLM from scratch" ch. 36.3,
capacity and overflow: a rejected path may be rerouted, calling another
expert's parameters; vegetog "MoE token routing" sec. 5: an over-capacity
token is dropped from that expert's branch or rerouted, depending on the
implementation).

Reading pinned here: a token's rerouting candidates are its next-ranked
experts (ranks k, k+1, ...), each weighted as the router's normalisation
weights it against the token's chosen set; after Algorithm 36.1's token-order
acceptance, rejected paths fill the slots left free in rounds, each taking
its token's next candidate that was not full at the round's start, offers
accepted in token order.

Each test checks against the page's worked example, a hand-derived closed
form, an invariant, or a second implementation of the rule written
differently (a per-expert queue simulation) on tiny random inputs.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _golden, _frac, _n4_setup


def _route_scores(P):
    """One-hot tokens with scores ln P: the router's probabilities are P."""
    N, E = P.shape
    x = np.eye(N, dtype=np.float32)
    W_r = np.log(np.asarray(P, np.float64)).T.astype(np.float32)
    return x, W_r


def _linear_outputs(ids2, w2, slot2, N):
    """Y_t = sum over served paths of weight * (e + 1): the page's linear
    experts F_e(x) = e x (1-based) on one-hot tokens, read on the diagonal."""
    y = np.zeros(N)
    for t in range(N):
        for j in range(ids2.shape[1]):
            if ids2[t, j] >= 0 and slot2[t, j] >= 0:
                y[t] += w2[t, j] * (ids2[t, j] + 1)
    return y


def _run(P, k, C, X, norm):
    x, W_r = _route_scores(P)
    r = oracle.route(x, W_r, k=k, norm=norm)
    cand, cw = oracle.reroute_candidates(r["logits"], r["ids"], r["invalid"], k, X, norm)
    dr = oracle.dispatch_reroute(r["ids"], cand, P.shape[1], C)
    ids2, w2, slot2 = oracle.served_records(r["ids"], r["w"], dr["slot"], dr["rr_e"], dr["rr_slot"],
                                            dr["rr_q"], cw)
    return r, cand, cw, dr, _linear_outputs(ids2, w2, slot2, P.shape[0])


def test_page_example_reroute_finds_no_free_expert():
    # ch. 36.4: N = 4, E_r = 3, k = 2, C = 3.  Token 4's path to expert 2 is
    # rejected; its only other expert (expert 1, rank 3) already holds C = 3
    # rows, so the path still adds 0: y_4 = 7/3 x_4, as under the zero policy.
    g, x, W_r = _n4_setup()
    P = np.array(g["probabilities"])
    C = g["capacity"]
    r, cand, cw, dr, y = _run(P, 2, C, 1, oracle.NORM_RENORM)
    np.testing.assert_array_equal(cand[:, 0], [2, 2, 2, 0])      # each token's third-ranked expert
    assert dr["stats"]["rerouted"] == 0 and dr["stats"]["rejected"] == 1 and dr["stats"]["rounds"] == 0
    np.testing.assert_array_equal(dr["rr_e"], -1)
    assert list(dr["acc"]) == g["accepted_loads"]
    assert abs(y[3] - _frac(g["token4_output_coefficient_zero_reject"])) < 1e-6
    for t in range(3):
        assert abs(y[t] - _frac(g["uncapped_output_coefficients"][t])) < 1e-6
    # same first-choice slots as Algorithm 36.1
    np.testing.assert_array_equal(dr["slot"], oracle.dispatch(r["ids"], E=3, C=C)["slot"])


def test_reroute_to_second_choice_full_probability():
    # three tokens all prefer expert 0 (C = 1, k = 1, Switch weights p):
    # token 0 keeps it; tokens 1 and 2 move to their second choices in one
    # round: y = (0.6 * 1, 0.4 * 2, 0.3 * 3)
    P = np.array([[0.6, 0.3, 0.1], [0.5, 0.4, 0.1], [0.5, 0.2, 0.3]])
    r, cand, cw, dr, y = _run(P, 1, 1, 2, oracle.NORM_FULLPROB)
    np.testing.assert_array_equal(dr["rr_e"][:, 0], [-1, 1, 2])
    np.testing.assert_array_equal(dr["rr_slot"][:, 0], [-1, 0, 0])
    assert dr["stats"]["rerouted"] == 2 and dr["stats"]["rounds"] == 1 and dr["stats"]["rejected"] == 0
    np.testing.assert_allclose(y, [0.6, 0.8, 0.9], rtol=0, atol=1e-6)


def test_reroute_competition_takes_a_second_round():
    # tokens 1 and 2 both rank expert 1 second: token 1 wins it in round 1
    # (token order); token 2 is refused and takes expert 2 in round 2
    P = np.array([[0.6, 0.3, 0.1], [0.5, 0.4, 0.1], [0.5, 0.4, 0.1]])
    r, cand, cw, dr, y = _run(P, 1, 1, 2, oracle.NORM_FULLPROB)
    np.testing.assert_array_equal(dr["rr_e"][:, 0], [-1, 1, 2])
    np.testing.assert_array_equal(dr["rr_q"][:, 0], [-1, 0, 1])
    assert dr["stats"]["rounds"] == 2
    np.testing.assert_allclose(y, [0.6, 0.8, 0.3], rtol=0, atol=1e-6)
    # with one candidate only, token 2 has nowhere to go
    r1, _, _, dr1, y1 = _run(P, 1, 1, 1, oracle.NORM_FULLPROB)
    np.testing.assert_array_equal(dr1["rr_e"][:, 0], [-1, 1, -1])
    assert dr1["stats"]["tokens_skipped"] == 1
    np.testing.assert_allclose(y1, [0.6, 0.8, 0.0], rtol=0, atol=1e-6)


def test_reroute_weights_under_renormalisation():
    # k = 2, C = 1: token 1 loses both first choices {0, 1}; its candidates are
    # experts 2 and 3 with weights p / (p_0 + p_1) = 2/7 and 1/7:
    # y_1 = 2/7 * 3 + 1/7 * 4 = 10/7
    P = np.array([[0.4, 0.3, 0.2, 0.1], [0.4, 0.3, 0.2, 0.1]])
    r, cand, cw, dr, y = _run(P, 2, 1, 2, oracle.NORM_RENORM)
    np.testing.assert_array_equal(cand[1], [2, 3])
    np.testing.assert_allclose(cw[1], [2 / 7, 1 / 7], rtol=0, atol=1e-6)
    np.testing.assert_array_equal(dr["rr_e"][1], [2, 3])
    assert abs(y[0] - (4 / 7 * 1 + 3 / 7 * 2)) < 1e-6
    assert abs(y[1] - 10 / 7) < 1e-6


def test_skip_experts_full_at_round_start():
    # token 2's first candidate (expert 1) is full before rerouting starts
    # (token 1 chose it first), so the token goes straight to expert 2
    P = np.array([[0.7, 0.2, 0.1], [0.2, 0.7, 0.1], [0.6, 0.3, 0.1]])
    r, cand, cw, dr, y = _run(P, 1, 1, 2, oracle.NORM_FULLPROB)
    np.testing.assert_array_equal(r["ids"][:, 0], [0, 1, 0])
    np.testing.assert_array_equal(dr["rr_e"][:, 0], [-1, -1, 2])
    np.testing.assert_array_equal(dr["rr_q"][:, 0], [-1, -1, 1])
    assert dr["stats"]["rounds"] == 1


def _queue_reference(ids, cand, E, C):
    """The rule written differently: per round, every expert keeps a queue of
    (token, path, candidate index) offers built from a snapshot of which
    experts are full; queues are served in token order."""
    N, k = ids.shape
    X = cand.shape[1]
    load = np.zeros(E, int)
    slot = -np.ones((N, k), int)
    for t in range(N):
        for j in range(k):
            e = ids[t, j]
            if e >= 0:
                if load[e] < C:
                    slot[t, j] = load[e]
                load[e] += 1
    rows = np.minimum(load, C)
    rr = -np.ones((N, k), int)
    rs = -np.ones((N, k), int)
    ptr = [0] * N
    while True:
        full = {e for e in range(E) if rows[e] >= C}
        queues = {e: [] for e in range(E)}
        for t in range(N):
            for j in range(k):
                if ids[t, j] < 0 or slot[t, j] >= 0 or rr[t, j] >= 0:
                    continue
                while ptr[t] < X and cand[t, ptr[t]] >= 0 and cand[t, ptr[t]] in full:
                    ptr[t] += 1
                if ptr[t] < X and cand[t, ptr[t]] >= 0:
                    queues[cand[t, ptr[t]]].append((t, j))
                    ptr[t] += 1
        if not any(queues.values()):
            return slot, rr, rs, rows
        for e, q in queues.items():
            for t, j in sorted(q):
                if rows[e] < C:
                    rr[t, j], rs[t, j] = e, rows[e]
                    rows[e] += 1


@pytest.mark.parametrize("seed", range(6))
def test_reroute_matches_queue_simulation_and_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    N, E = int(rng.integers(5, 40)), int(rng.integers(3, 9))
    k = int(rng.integers(1, min(3, E - 1) + 1))
    X = int(rng.integers(1, E - k + 1))
    # skewed scores so that a few experts overflow
    g = rng.standard_normal((N, E)) - 0.6 * np.arange(E)[None, :]
    P = np.exp(g) / np.exp(g).sum(axis=1, keepdims=True)
    C = max(1, int(rng.integers(1, max(2, N * k // E + 1))))
    norm = [oracle.NORM_RENORM, oracle.NORM_FULLPROB][seed % 2]
    r, cand, cw, dr, _ = _run(P, k, C, X, norm)
    slot, rr, rs, rows = _queue_reference(r["ids"], cand, E, C)
    np.testing.assert_array_equal(dr["slot"], slot)
    np.testing.assert_array_equal(dr["rr_e"], rr)
    np.testing.assert_array_equal(dr["rr_slot"], rs)
    np.testing.assert_array_equal(dr["acc"], rows)
    assert (dr["acc"] <= C).all()
    for e in range(E):   # every expert's slots 0..acc-1 are used exactly once
        used = sorted(list(dr["slot"][r["ids"] == e][dr["slot"][r["ids"] == e] >= 0]) +
                      list(dr["rr_slot"][dr["rr_e"] == e]))
        assert used == list(range(dr["acc"][e]))
    for t in range(N):
        mine = [e for e in r["ids"][t] if e >= 0] + [e for e in dr["rr_e"][t] if e >= 0]
        assert len(mine) == len(set(mine))                         # never two paths on one expert
        for j in range(k):
            if dr["rr_e"][t, j] >= 0:                              # rerouted to a candidate ...
                assert dr["rr_e"][t, j] == cand[t, dr["rr_q"][t, j]]
                assert dr["rr_e"][t, j] not in r["ids"][t]         # ... outside the chosen set
        unserved = [(j) for j in range(k) if r["ids"][t, j] >= 0 and dr["slot"][t, j] < 0 and dr["rr_e"][t, j] < 0]
        if unserved:   # maximal: every candidate the token did not use is full
            for q in range(X):
                e = cand[t, q]
                if e >= 0 and e not in dr["rr_e"][t]:
                    assert dr["acc"][e] == C
    # candidates are the next-ranked experts, weighted against the chosen set
    for t in range(N):
        order = sorted(range(E), key=lambda e: (-r["logits"][t, e], e))
        np.testing.assert_array_equal(cand[t], (order[k:k + X] + [-1] * X)[:X])
        p = np.exp(r["logits"][t] - r["logits"][t].max())
        p /= p.sum()
        den = p[r["ids"][t]].sum() if norm == oracle.NORM_RENORM else 1.0
        np.testing.assert_allclose(cw[t, :min(X, E - k)], p[order[k:k + X]] / den, rtol=1e-12)
    st = dr["stats"]
    assert st["requested"] == N * k and st["accepted"] == int(dr["acc"].sum())
    assert st["rerouted"] == int((dr["rr_e"] >= 0).sum())


def test_reroute_without_overflow_equals_algorithm_36_1():
    rng = np.random.default_rng(3)
    N, E, k = 50, 6, 2
    P = rng.dirichlet(np.ones(E), size=N)
    r, cand, cw, dr, _ = _run(P, k, N, 3, oracle.NORM_RENORM)
    d0 = oracle.dispatch(r["ids"], E=E, C=N)
    np.testing.assert_array_equal(dr["slot"], d0["slot"])
    assert (dr["rr_e"] < 0).all() and dr["stats"]["rerouted"] == 0


def test_forward_with_reroute_matches_dense_masked_evaluation():
    """The whole layer under rerouting against a dense evaluation: every
    expert on every token (numpy products), masked by the served paths'
    weights from the queue simulation."""
    rng = np.random.default_rng(21)
    N, d, d_f, E, k, X = 40, 12, 10, 6, 2, 3
    x = rng.standard_normal((N, d)).astype(np.float32)
    W_r = (rng.standard_normal((E, d)) / math.sqrt(d)).astype(np.float32)
    b = (-0.8 * np.arange(E)).astype(np.float32)    # low indices hot: overflow
    Wg = (rng.standard_normal((E, d_f, d)) / math.sqrt(d)).astype(np.float32)
    Wu = (rng.standard_normal((E, d_f, d)) / math.sqrt(d)).astype(np.float32)
    Wd = (rng.standard_normal((E, d, d_f)) / math.sqrt(d_f)).astype(np.float32)
    c = 0.9
    out = oracle.forward(x, W_r, Wg, Wu, Wd, k=k, norm=oracle.NORM_RENORM, c=c, b_r=b, reject_policy=2,
                         reroute_depth=X)
    C = oracle.capacity(c, N, k, E)
    assert out["stats"]["rerouted"] > 0
    x64 = x.astype(np.float64)
    g = x64 @ W_r.astype(np.float64).T + b.astype(np.float64)
    p = np.exp(g - g.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ids = np.array([sorted(range(E), key=lambda e: (-g[t, e], e))[:k] for t in range(N)])
    cand = np.array([sorted(range(E), key=lambda e: (-g[t, e], e))[k:k + X] for t in range(N)])
    slot, rr, rs, rows = _queue_reference(ids, cand, E, C)
    A = np.zeros((N, E))
    for t in range(N):
        den = p[t, ids[t]].sum()
        for j in range(k):
            if slot[t, j] >= 0:
                A[t, ids[t, j]] = p[t, ids[t, j]] / den
            if rr[t, j] >= 0:
                A[t, rr[t, j]] = p[t, rr[t, j]] / den
    Y = np.zeros((N, d))
    for e in range(E):
        G = x64 @ Wg[e].astype(np.float64).T
        U = x64 @ Wu[e].astype(np.float64).T
        Y += A[:, e:e + 1] * ((G / (1 + np.exp(-G)) * U) @ Wd[e].astype(np.float64).T)
    np.testing.assert_allclose(out["Y"], Y, rtol=1e-12, atol=1e-12)
