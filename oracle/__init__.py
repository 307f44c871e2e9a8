"""CPU oracle of the sparse-MoE layer forward pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product path never
does.  It shares no code with the CUDA library; both sides read the same
seeded inputs from ``seeded_inputs``.

The arithmetic lives in ``oracle.c`` (plain C, double precision); this module
marshals numpy arrays and adds the host-side definitions that are exact in
rational arithmetic (capacity, statistics, parameter counts).

Parity status per function (what pins it, see tests/test_oracle_pins.py):
  capacity       pinned: C=160, C=157, C=3 printed on the pages; C=640 closed form
  route RENORM   pinned: 4-expert example weights 0.6/0.4; N=4,E_r=3,k=2 table
  route FULLPROB pinned: closed form a = p (x = 0 gives 1/E_r)
  route WLR      the pages print no worked numbers: pinned only by hand-derived
                 tiny cases and the theta = 0 limit (no pruning)
  dispatch/stats pinned: N=4 example loads (3,4,1), accepted (3,3,1), reject
                 rate 1/8, tokens affected 1/4, rho_max = 1.5; invariants
  combine        pinned: y = [4.4, 2.8]; outputs 11/9, 4/3, 25/18, 25/9, 7/3
  swiglu         pinned: closed forms on 1-wide experts; brute-force dense check
  forward        pinned: dense all-expert evaluation with masked weights
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from fractions import Fraction

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

NORM_RENORM, NORM_FULLPROB, NORM_WLR = 0, 1, 2
DT_F32, DT_BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so beside it (gcc -O2, OpenMP)."""
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, src, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None
_P = ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_route.argtypes = [i64, i32, i32, i32, i32, dbl, i32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_dispatch.argtypes = [i64, i32, i32, i64, _P, _P, _P, _P, _P]
        lib.oracle_dispatch_ranked.argtypes = [i64, i32, i32, i64, _P, _P, _P, _P, _P, _P]
        lib.oracle_dispatch_priority.argtypes = [i64, i32, i32, i64, _P, _P, _P, _P, _P, _P]
        lib.oracle_swiglu_dense.argtypes = [i32, i32, i32, i32, _P, i64, _P, _P, _P, _P]
        lib.oracle_swiglu_rows.argtypes = [i32, i32, i32, i32, _P, _P, i64, _P, _P, _P, _P]
        lib.oracle_combine.argtypes = [i64, i32, i32, _P, _P, _P, _P, _P]
        lib.oracle_forward_rows.argtypes = [i32, i32, i32, i32, i32, i32, _P, _P, _P, _P, _P, i64,
                                            _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_reject_weights.argtypes = [i64, i32, i32, _P, _P, _P, _P]
        lib.oracle_forward.argtypes = [i64, i32, i32, i32, i32, i32, dbl, i32, i64, i32, i32, i32,
                                       _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                       _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_reroute_candidates.argtypes = [i64, i32, i32, i32, i32, _P, _P, _P, _P, _P]
        lib.oracle_dispatch_reroute.argtypes = [i64, i32, i32, i64, i32, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_round_bf16.argtypes = [dbl]
        lib.oracle_round_bf16.restype = dbl
        for f in ("oracle_route", "oracle_dispatch", "oracle_dispatch_ranked", "oracle_reject_weights",
                  "oracle_reroute_candidates", "oracle_dispatch_reroute",
                  "oracle_swiglu_rows", "oracle_combine",
                  "oracle_forward_rows", "oracle_forward"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _dtype_of(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return DT_BF16
    if a.dtype == np.float32:
        return DT_F32
    raise TypeError(f"oracle inputs are fp32 or bf16 bit patterns (uint16), got {a.dtype}")


def _c(a, dt=None):
    if a is None:
        return None
    return np.ascontiguousarray(a if dt is None else a.astype(dt, copy=False))


# ---------------------------------------------------------------------------
# Exact host definitions
# ---------------------------------------------------------------------------
def capacity(c: float, N: int, k: int, E: int) -> int:
    """C = ceil(c * T * k / E) (review equations; ch. 36.3 eq. 36.13 with the
    capacity factor gamma; vegetog sec. 6 with k = 1), on the exact rational
    value of c.  When c*T*k/E lies within 1e-9 (relative) of an integer, that
    integer is taken, so that a decimal factor such as 1.1 whose binary value
    is a hair above 11/10 does not bump an exact integer up.  c <= 0 means no
    capacity limit: C = N, the largest load one expert can receive."""
    if c <= 0:
        return int(N)
    q = Fraction(c) * N * k / E
    r = round(q)
    if abs(q - r) <= Fraction(1, 10 ** 9) * max(1, q):
        C = int(r)
    else:
        C = math.ceil(q)
    return max(C, 1) if N > 0 else max(C, 0)


def rho_max(L: np.ndarray, N: int, k: int, E: int) -> float:
    """rho_max = max_e L_e / (T k / E) (review equations; ch. 36.4)."""
    if N == 0:
        return 0.0
    return float(Fraction(int(np.max(L))) / (Fraction(N * k, E)))


def load_percentile(L: np.ndarray, q: float) -> int:
    """Nearest-rank percentile of the per-expert requested loads (the tail
    statistics the review asks to report next to the maximum)."""
    s = np.sort(np.asarray(L, dtype=np.int64))
    if s.size == 0:
        return 0
    rank = max(1, math.ceil(q / 100.0 * s.size))
    return int(s[rank - 1])


def param_counts(d: int, d_f: int, E: int, k: int, L: int = 1):
    """SwiGLU expert parameters P_e = 3 d d_f (no bias), all routed experts
    L E P_e and the routed parameters active per token L k P_e (ch. 36.5;
    vegetog sec. 4)."""
    Pe = 3 * d * d_f
    return Pe, L * E * Pe, L * k * Pe


# ---------------------------------------------------------------------------
# Wrappers of the C oracle
# ---------------------------------------------------------------------------
def route(x, W_r, k: int, norm: int, theta: float = 0.0, b_r=None, lat=None):
    """Router scores, softmax, top-k and weights (see oracle.c).  Returns a
    dict with ids [N,k] int32, w [N,k] f64, margin [N], wlr_gap [N],
    invalid [N] bool and logits [N,E] f64."""
    x, W_r = _c(x), _c(W_r)
    dt = _dtype_of(x)
    assert _dtype_of(W_r) == dt
    N, d = x.shape
    E = W_r.shape[0]
    ids = np.empty((N, k), np.int32)
    w = np.empty((N, k), np.float64)
    margin = np.empty(N, np.float64)
    gap = np.empty(N, np.float64)
    inv = np.empty(N, np.uint8)
    logits = np.empty((N, E), np.float64)
    b = _c(b_r, np.float32)
    la = _c(lat, np.float32)
    rc = _load().oracle_route(N, d, E, k, norm, theta, dt, _ptr(x), _ptr(W_r), _ptr(b), _ptr(la),
                              _ptr(logits), _ptr(ids), _ptr(w), _ptr(margin), _ptr(gap), _ptr(inv))
    if rc:
        raise ValueError("oracle_route: invalid arguments")
    return {"ids": ids, "w": w, "margin": margin, "wlr_gap": gap, "invalid": inv.astype(bool),
            "logits": logits}


def dispatch(ids, E: int, C: int):
    """Token-order acceptance under capacity C (Algorithm 36.1).  Returns slot
    [N,k] int32, L [E], acc [E] and the counters of oracle_dispatch."""
    ids = _c(ids, np.int32)
    N, k = ids.shape
    slot = np.empty((N, k), np.int32)
    L = np.empty(E, np.int64)
    acc = np.empty(E, np.int64)
    cnt = np.empty(7, np.int64)
    rc = _load().oracle_dispatch(N, k, E, C, _ptr(ids), _ptr(slot), _ptr(L), _ptr(acc), _ptr(cnt))
    if rc:
        raise ValueError("oracle_dispatch: invalid arguments")
    names = ("requested", "accepted", "rejected", "O", "tokens_affected", "tokens_skipped", "L_max")
    stats = {n: int(v) for n, v in zip(names, cnt)}
    return {"slot": slot, "L": L, "acc": acc, "stats": stats}


def dispatch_priority(ids, w, E: int, C: int):
    """Acceptance by routing weight: each expert keeps the C requests with the
    largest weight (equal weights: earlier token); accepted rows in token
    order (see oracle.c).  Same return values as dispatch."""
    ids = _c(ids, np.int32)
    N, k = ids.shape
    wd = _c(np.asarray(w, np.float64).reshape(N, k), np.float64)
    slot = np.empty((N, k), np.int32)
    L = np.empty(E, np.int64)
    acc = np.empty(E, np.int64)
    cnt = np.empty(7, np.int64)
    rc = _load().oracle_dispatch_priority(N, k, E, C, _ptr(ids), _ptr(wd), _ptr(slot), _ptr(L), _ptr(acc),
                                          _ptr(cnt))
    if rc:
        raise ValueError("oracle_dispatch_priority: invalid arguments")
    names = ("requested", "accepted", "rejected", "O", "tokens_affected", "tokens_skipped", "L_max")
    stats = {n: int(v) for n, v in zip(names, cnt)}
    return {"slot": slot, "L": L, "acc": acc, "stats": stats}


def dispatch_ranked(ids, E: int, C: int, base):
    """Acceptance for one rank's shard of a routing group split over ranks
    in token order; base[e] = requests for e by earlier ranks (see oracle.c).
    Returns slot (group-wide slot or -1), this shard's L and acc, and the
    shard's counters."""
    ids = _c(ids, np.int32)
    N, k = ids.shape
    b = _c(np.asarray(base), np.int64)
    slot = np.empty((N, k), np.int32)
    L = np.empty(E, np.int64)
    acc = np.empty(E, np.int64)
    cnt = np.empty(7, np.int64)
    rc = _load().oracle_dispatch_ranked(N, k, E, C, _ptr(ids), _ptr(b), _ptr(slot), _ptr(L), _ptr(acc),
                                        _ptr(cnt))
    if rc:
        raise ValueError("oracle_dispatch_ranked: invalid arguments")
    names = ("requested", "accepted", "rejected", "O", "tokens_affected", "tokens_skipped", "L_max")
    return {"slot": slot, "L": L, "acc": acc, "stats": {n: int(v) for n, v in zip(names, cnt)}}


def reroute_candidates(logits, ids, invalid, k: int, X: int, norm: int):
    """Each token's next-ranked experts (ranks k .. k+X-1, -1 past E_r) and
    their weights under the layer's normalisation against the token's chosen
    set (see oracle.c, rerouting as an overflow policy).  logits [N, E] f64,
    ids [N, k], invalid [N] bool.  Returns (cand [N, X] int32, cand_w [N, X] f64)."""
    lg = _c(np.asarray(logits, np.float64))
    N, E = lg.shape
    ids = _c(ids, np.int32)
    inv = _c(np.asarray(invalid, np.uint8))
    cand = np.empty((N, X), np.int32)
    cw = np.empty((N, X), np.float64)
    rc = _load().oracle_reroute_candidates(N, E, k, X, norm, _ptr(lg), _ptr(ids), _ptr(inv), _ptr(cand), _ptr(cw))
    if rc:
        raise ValueError("oracle_reroute_candidates: invalid arguments")
    return cand, cw


def dispatch_reroute(ids, cand, E: int, C: int):
    """Token-order acceptance with rerouting of rejected paths to each token's
    next-ranked experts with free slots, in rounds (see oracle.c).  Returns
    slot (first choice), rr_e, rr_slot, rr_q [N, k], L (first-choice loads),
    acc (rows per expert, rerouted included) and the statistics."""
    ids = _c(ids, np.int32)
    cand = _c(cand, np.int32)
    N, k = ids.shape
    X = cand.shape[1]
    slot = np.empty((N, k), np.int32)
    rr_e = np.empty((N, k), np.int32)
    rr_slot = np.empty((N, k), np.int32)
    rr_q = np.empty((N, k), np.int32)
    L = np.empty(E, np.int64)
    acc = np.empty(E, np.int64)
    cnt = np.empty(9, np.int64)
    rc = _load().oracle_dispatch_reroute(N, k, E, C, X, _ptr(ids), _ptr(cand), _ptr(slot), _ptr(rr_e),
                                         _ptr(rr_slot), _ptr(rr_q), _ptr(L), _ptr(acc), _ptr(cnt))
    if rc:
        raise ValueError("oracle_dispatch_reroute: invalid arguments")
    names = ("requested", "accepted", "rejected", "O", "tokens_affected", "tokens_skipped", "L_max",
             "rerouted", "rounds")
    return {"slot": slot, "rr_e": rr_e, "rr_slot": rr_slot, "rr_q": rr_q, "L": L, "acc": acc,
            "stats": {n: int(v) for n, v in zip(names, cnt)}}


def served_records(ids, w, slot, rr_e, rr_slot, rr_q, cand_w):
    """The paths that run an expert, as [N, 2k] records for forward_rows:
    columns 0..k-1 the first-choice paths (weight a_te, slot or -1), columns
    k..2k-1 the rerouted paths (their candidate's weight, slot or -1)."""
    ids = np.asarray(ids, np.int32)
    N, k = ids.shape
    rr_e = np.asarray(rr_e, np.int32)
    rq = np.asarray(rr_q)
    cw = np.asarray(cand_w, np.float64)
    w_rr = np.where(rq >= 0, cw[np.arange(N)[:, None], np.maximum(rq, 0)], 0.0)
    ids2 = np.concatenate([ids, rr_e], axis=1).astype(np.int32)
    w2 = np.concatenate([np.asarray(w, np.float64), w_rr], axis=1)
    slot2 = np.concatenate([np.asarray(slot, np.int32), np.asarray(rr_slot, np.int32)], axis=1)
    return ids2, w2, slot2


def swiglu_rows(x, rows, Wg, Wu, Wd, round_h=None):
    """E(x_t) for t in rows, for one expert with weights Wg, Wu [d_f, d] and
    Wd [d, d_f].  Returns [len(rows), d] float64."""
    x, Wg, Wu, Wd = _c(x), _c(Wg), _c(Wu), _c(Wd)
    dt = _dtype_of(x)
    d = x.shape[1]
    d_f = Wg.shape[0]
    rows = _c(np.asarray(rows), np.int64)
    out = np.empty((rows.size, d), np.float64)
    if round_h is None:
        round_h = dt == DT_BF16
    _load().oracle_swiglu_rows(d, d_f, dt, int(bool(round_h)), _ptr(x), _ptr(rows), rows.size,
                               _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(out))
    return out


def combine(ids, w, slot, H_per_expert, d: int):
    """Y_t = sum over accepted records of a_te H_e[slot] (Algorithm 36.1, last
    step).  H_per_expert: list (length E) of [rows, d] float64 arrays or None."""
    ids = _c(ids, np.int32)
    w = _c(w, np.float64)
    slot = _c(slot, np.int32)
    N, k = ids.shape
    keep = [None if h is None else _c(h, np.float64) for h in H_per_expert]
    table = (ctypes.c_void_p * len(keep))(*[(0 if h is None else h.ctypes.data) for h in keep])
    Y = np.empty((N, d), np.float64)
    _load().oracle_combine(N, k, d, _ptr(ids), _ptr(w), _ptr(slot), ctypes.cast(table, ctypes.c_void_p),
                           _ptr(Y))
    return Y


def forward_rows(x, ids, w, slot, tokens, Wg, Wu, Wd, Ws=None):
    """Output rows Y_t for the given tokens from routing records (ids, w,
    slot) and the stacked expert weights; Ws = (Ws_g, Ws_u, Ws_d) adds the
    shared expert.  Returns [len(tokens), d] float64."""
    x, Wg, Wu, Wd = _c(x), _c(Wg), _c(Wu), _c(Wd)
    dt = _dtype_of(x)
    N, d = x.shape
    E, d_f = Wg.shape[0], Wg.shape[1]
    ids, w, slot = _c(ids, np.int32), _c(w, np.float64), _c(slot, np.int32)
    k = ids.shape[1]
    tokens = _c(np.asarray(tokens), np.int64)
    Y = np.empty((tokens.size, d), np.float64)
    if Ws is not None and Ws[0] is not None:
        Wsg, Wsu, Wsd = (_c(a) for a in Ws)
        dsh = Wsg.shape[0]
    else:
        Wsg = Wsu = Wsd = None
        dsh = 0
    _load().oracle_forward_rows(d, d_f, E, k, dt, dsh, _ptr(x), _ptr(ids), _ptr(w), _ptr(slot),
                                _ptr(tokens), tokens.size, _ptr(Wg), _ptr(Wu), _ptr(Wd),
                                _ptr(Wsg), _ptr(Wsu), _ptr(Wsd), _ptr(Y))
    return Y


def reject_weights(ids, w, slot, policy: int):
    """Combine weights of the routing records under an overflow policy
    (0: zero, no renormalisation; 1: accepted paths of a token that lost a
    path rescaled to sum to one); see oracle.c."""
    ids = _c(ids, np.int32)
    N, k = ids.shape
    w = _c(w, np.float64)
    slot = _c(slot, np.int32)
    wc = np.empty((N, k), np.float64)
    _load().oracle_reject_weights(N, k, int(policy), _ptr(ids), _ptr(w), _ptr(slot), _ptr(wc))
    return wc


def forward(x, W_r, Wg, Wu, Wd, *, k: int, norm: int, c: float = 0.0, theta: float = 0.0,
            b_r=None, lat=None, Ws=None, reject_policy: int = 0, accept_order: int = 0,
            reroute_depth: int = 0):
    """The whole layer (Algorithm 36.1 generalised by the weighting mode and a
    shared expert).  Returns a dict with Y [N,d] f64, the routing records,
    per-expert loads and the statistics.  reject_policy 2 reroutes rejected
    paths to up to reroute_depth next-ranked experts per token (token-order
    acceptance only)."""
    x, W_r, Wg, Wu, Wd = _c(x), _c(W_r), _c(Wg), _c(Wu), _c(Wd)
    dt = _dtype_of(x)
    N, d = x.shape
    E, d_f = Wg.shape[0], Wg.shape[1]
    C = capacity(c, N, k, E)
    if reject_policy == 2:
        return _forward_reroute(x, W_r, Wg, Wu, Wd, k=k, norm=norm, C=C, b_r=b_r, Ws=Ws,
                                depth=reroute_depth)
    Y = np.zeros((N, d), np.float64)
    ids = np.empty((N, k), np.int32)
    w = np.empty((N, k), np.float64)
    slot = np.empty((N, k), np.int32)
    margin = np.empty(N, np.float64)
    gap = np.empty(N, np.float64)
    inv = np.empty(N, np.uint8)
    L = np.empty(E, np.int64)
    acc = np.empty(E, np.int64)
    cnt = np.empty(7, np.int64)
    if Ws is not None and Ws[0] is not None:
        Wsg, Wsu, Wsd = (_c(a) for a in Ws)
        dsh = Wsg.shape[0]
    else:
        Wsg = Wsu = Wsd = None
        dsh = 0
    b = _c(b_r, np.float32)
    la = _c(lat, np.float32)
    rc = _load().oracle_forward(N, d, d_f, E, k, norm, theta, dt, max(C, 1), dsh, int(reject_policy),
                                int(accept_order),
                                _ptr(x), _ptr(W_r),
                                _ptr(b), _ptr(la), _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(Wsg), _ptr(Wsu),
                                _ptr(Wsd), _ptr(Y), _ptr(ids), _ptr(w), _ptr(slot), _ptr(margin),
                                _ptr(gap), _ptr(inv), _ptr(L), _ptr(acc), _ptr(cnt))
    if rc:
        raise ValueError("oracle_forward: invalid arguments")
    names = ("requested", "accepted", "rejected", "O", "tokens_affected", "tokens_skipped", "L_max")
    stats = {n: int(v) for n, v in zip(names, cnt)}
    stats["C"] = C
    stats["rho_max"] = rho_max(L, N, k, E) if N else 0.0
    return {"Y": Y, "ids": ids, "w": w, "slot": slot, "margin": margin, "wlr_gap": gap,
            "invalid": inv.astype(bool), "L": L, "acc": acc, "stats": stats, "C": C}


def _forward_reroute(x, W_r, Wg, Wu, Wd, *, k, norm, C, b_r, Ws, depth):
    """forward() under rerouting: route, each token's candidates, token-order
    acceptance with rerouting rounds, then every served path's expert output
    weighted and summed per token (plus the shared expert)."""
    N, d = x.shape
    E = Wg.shape[0]
    r = route(x, W_r, k=k, norm=norm, b_r=b_r)
    cand, cw = reroute_candidates(r["logits"], r["ids"], r["invalid"], k, depth, norm)
    dr = dispatch_reroute(r["ids"], cand, E, C)
    ids2, w2, slot2 = served_records(r["ids"], r["w"], dr["slot"], dr["rr_e"], dr["rr_slot"], dr["rr_q"], cw)
    Y = forward_rows(x, ids2, w2, slot2, np.arange(N), Wg, Wu, Wd, Ws=Ws) if N else np.zeros((0, d))
    stats = dict(dr["stats"])
    stats["C"] = C
    stats["rho_max"] = rho_max(dr["L"], N, k, E) if N else 0.0
    return {"Y": Y, "ids": r["ids"], "w": r["w"], "slot": dr["slot"], "margin": r["margin"],
            "wlr_gap": r["wlr_gap"], "invalid": r["invalid"], "L": dr["L"], "acc": dr["acc"], "stats": stats,
            "C": C, "cand": cand, "cand_w": cw, "rr_e": dr["rr_e"], "rr_slot": dr["rr_slot"], "rr_q": dr["rr_q"]}


def expert_choice(x, W_r, Wg, Wu, Wd, C: int, b_r=None, P=None):
    """Expert-choice routing ("LLM from scratch" ch. 36.6, table of routing
    styles: each expert picks a limited number of tokens by its column of
    scores; a token may be picked by several experts or by none), written out
    from that definition: P = softmax over experts of x W_r^T + b; expert e
    takes the C tokens with the largest P[t, e] (equal scores: the lower token
    index); Y_t = sum over the experts that took t of P[t, e] E_e(x_t).
    P may be given (for example the scores another implementation computed)
    so that both sides pick by the same numbers.  Returns Y [N, d] float64,
    the picks [E, C'] (token indices, C' = min(C, N)) and P."""
    x = _c(x)
    dt = _dtype_of(x)
    N, d = x.shape
    E = Wg.shape[0]
    if P is None:
        r = route(x, W_r, k=E, norm=NORM_FULLPROB, b_r=b_r)
        G = r["logits"]
        G = G - G.max(axis=1, keepdims=True)
        P = np.exp(G)
        P /= P.sum(axis=1, keepdims=True)
    P = np.asarray(P, np.float64)
    Y = np.zeros((N, d), np.float64)
    picks = []
    for e in range(E):
        order = sorted(range(N), key=lambda t: (-P[t, e], t))[:min(C, N)]
        picks.append(order)
        if order:
            out = swiglu_rows(x, order, Wg[e], Wu[e], Wd[e])
            for row, t in zip(out, order):
                Y[t] += P[t, e] * row
    return {"Y": Y, "picks": np.array(picks, np.int64), "P": P}


def soft_moe(x, Phi, Wg, Wu, Wd, p: int):
    """Soft MoE ("LLM from scratch" ch. 36.6, Soft Mixture of Experts), written
    out from its definition: S = E_r p slots, slot e p + i belongs to expert e;
    scores Z = X Phi^T [N, S] (Phi stored [S, d]); dispatch weights D =
    softmax of Z over the tokens (each column sums to one); combine weights
    C = softmax of Z over the slots (each row sums to one); slot inputs
    Xs = D^T X [S, d]; slot outputs Ys_s = E_{e(s)}(Xs_s) (h rounded to bf16
    for bf16 weights, as in the other layers); Y = C Ys [N, d].  Returns Y,
    D, C, Xs and Ys in float64."""
    x, Phi, Wg, Wu, Wd = _c(x), _c(Phi), _c(Wg), _c(Wu), _c(Wd)
    dt = _dtype_of(x)
    X = _as_f64(x)
    F = _as_f64(Phi)
    N, d = X.shape
    E, d_f = Wg.shape[0], Wg.shape[1]
    S = E * p
    assert F.shape == (S, d)
    Z = X @ F.T
    D = np.exp(Z - Z.max(axis=0, keepdims=True))
    D /= D.sum(axis=0, keepdims=True)
    Cw = np.exp(Z - Z.max(axis=1, keepdims=True))
    Cw /= Cw.sum(axis=1, keepdims=True)
    Xs = D.T @ X
    Ys = np.empty((S, d), np.float64)
    for e in range(E):
        blk = np.ascontiguousarray(Xs[e * p:(e + 1) * p])
        out = np.empty((p, d), np.float64)
        _load().oracle_swiglu_dense(d, d_f, dt, int(dt == DT_BF16), _ptr(blk), p, _ptr(_c(Wg[e])),
                                    _ptr(_c(Wu[e])), _ptr(_c(Wd[e])), _ptr(out))
        Ys[e * p:(e + 1) * p] = out
    return {"Y": Cw @ Ys, "D": D, "C": Cw, "Xs": Xs, "Ys": Ys}


def _as_f64(a):
    """fp32 or bf16 (uint16 bit patterns) array -> float64, exactly."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def aux_balance(logits, ids, E: int, invalid=None) -> float:
    """The balance objective's value ("LLM from scratch" ch. 36.4, Switch's
    product of hard assignment shares and mean probabilities, top-k form):
    E_r sum_e f_e pbar_e with f_e = n_e / sum n (requests per expert before
    capacity; both f and pbar sum to one) and pbar_e the mean over the tokens
    with finite scores of the full-softmax probability p_te.  It equals one
    when both are uniform."""
    G = np.asarray(logits, np.float64)
    ok = ~np.asarray(invalid, bool) if invalid is not None else np.isfinite(G).all(axis=1)
    if not ok.any():
        return 0.0
    Gv = G[ok]
    P = np.exp(Gv - Gv.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    pbar = P.sum(axis=0) / ok.sum()
    ids = np.asarray(ids)
    n = np.bincount(ids[ids >= 0], minlength=E).astype(np.float64)
    if n.sum() == 0:
        return 0.0
    return float(E * ((n / n.sum()) * pbar).sum())


def round_bf16(v: float) -> float:
    return _load().oracle_round_bf16(float(v))


# gradients of the layer (numpy, float64): oracle/backward.py
from oracle.backward import (backward, bf16_round, combine_weights, expert_backward_columns,  # noqa: E402,F401
                             score_gradient, token_dx)
