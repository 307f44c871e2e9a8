"""CPU oracle of the sparse-MoE layer's gradients.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
the benchmark's CPU-baseline leg may import this module; it shares no code
with the CUDA library.

What it computes: the gradients of

    L = sum_{t,o} dY[t,o] Y[t,o]  +  aux_coef * aux

with respect to x, W_r, b_r, the expert weights and the shared expert's
weights, for the layer forward of this package ("LLM from scratch" ch. 36.3,
Algorithm 36.1: Y_t = sum over accepted paths of a_te E_e(x_t); ch. 36.6: the
shared expert adds F_sh(x_t) with weight 1; vegetog "MoE token routing"
sec. 3: the SwiGLU expert) and the balance objective of ch. 36.4
(aux = E_r sum_e f_e pbar_e).  The routing decisions -- the top-k sets, WLR
pruning and capacity acceptance -- are taken as given (``ids``, ``slot``):
they are piecewise constant in the inputs, so their derivative is zero almost
everywhere, and ch. 36.4 states that the hard counts f_e are held constant
while the mean probabilities pbar_e carry the gradient to the router through
the softmax Jacobian.

Every step is written out in float64 with numpy, one definition at a time:

  router   g_t = W_r x_t + b,  p_t = softmax(g_t)                (ch. 36.1)
  weights  RENORM and WLR survivors: a_j = m_j p_{e_j} / s,  s = sum over
           the token's chosen (surviving) experts of p;  m_j = 0 for an entry
           whose weight the forward set to 0 (WDMoE: a disconnected expert);
           FULLPROB: a_j = p_{e_j}                                (ch. 36.2)
  overflow policy 1 rescales a token's accepted weights to sum to one when it
           lost some but not all paths: wc_j = a_j / sum_acc a  (ch. 36.3-36.4)
  expert   z = W_g x, u = W_u x, h = SiLU(z) u, o = W_d h         (vegetog sec. 3)
  combine  Y_t = sum_acc wc_j o_j (+ shared)                      (Algorithm 36.1)

and their derivatives, by the chain rule:

  dwc_j = <dY_t, o_j>;   dh = wc_j W_d^T dY_t;   dW_d += wc_j dY_t h^T
  dz = dh u SiLU'(z),  SiLU'(z) = s(z) (1 + z (1 - s(z))),  s = logistic
  du = dh SiLU(z);     dx_t += W_g^T dz + W_u^T du;  dW_g += dz x^T;  dW_u += du x^T
  policy 1:  da_j = (dwc_j - sum_i dwc_i wc_i) / sum_acc a   (accepted j)
  RENORM / WLR:  dp_{e_j} = (m_j da_j - sum_i da_i a_i) / s
  FULLPROB:      dp_{e_j} = da_j
  softmax:   dg_e = p_e (dp_e - sum_i p_i dp_i)
  aux:       dg_te += aux_coef (E_r / N_valid) p_te (f_e - sum_i f_i p_ti),
             f = requests per expert / all requests, N_valid = tokens with
             finite scores (the same quantities as the objective's value)
  router:    dx_t += W_r^T dg_t,  dW_r = dg^T X,  db = sum_t dg_t

Precision contract of the bf16 layer (the storage precision of its
activations; the pages fix none for the backward): the upstream gradient dY
enters rounded to bf16; h is the forward's bf16-rounded activation (the
rounding passes the gradient through unchanged); the operands that the
weight-gradient and input-gradient contractions read are rounded to bf16:
do = bf16(wc dY) (for dW_d), dz and du.  Everything else is exact here.  The
fp32 layer rounds nothing.
"""
from __future__ import annotations

import numpy as np

NORM_RENORM, NORM_FULLPROB, NORM_WLR = 0, 1, 2


def bf16_round(v):
    """Each value rounded to the nearest bf16 number (8 significant bits,
    ties to even) from its exact double value: v = m 2^e with
    0.5 <= |m| < 1 has the quantum 2^(e-8), and 2^-133 below the normal
    range."""
    v = np.asarray(v, np.float64)
    _, e = np.frexp(v)
    q = np.maximum(e - 8, -133)
    return np.ldexp(np.rint(np.ldexp(v, -q)), q)


def _f64(a):
    """fp32 or bf16 (uint16 bit patterns) array -> float64, exactly."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _silu_parts(Z):
    s = 1.0 / (1.0 + np.exp(-Z))
    return Z * s, s * (1.0 + Z * (1.0 - s))


def _expert_backward(X, Wg, Wu, Wd, dYb, wc, rnd, round_h):
    """One expert on its rows X [R, d] with combine weights wc [R] and the
    upstream rows dYb [R, d].  Returns (dX, dWg, dWu, dWd, dwc)."""
    Z = X @ Wg.T
    U = X @ Wu.T
    S, dS = _silu_parts(Z)
    H = S * U
    if round_h:
        H = bf16_round(H)
    Gd = dYb @ Wd                         # W_d^T dY_t for every row  [R, d_f]
    dwc = (Gd * H).sum(axis=1)            # <dY_t, W_d h> = <W_d^T dY_t, h>
    dH = wc[:, None] * Gd
    dZ = rnd(dH * U * dS)
    dU = rnd(dH * S)
    dX = dZ @ Wg + dU @ Wu
    dWg = dZ.T @ X
    dWu = dU.T @ X
    dO = rnd(wc[:, None] * dYb)
    dWd = dO.T @ H
    return dX, dWg, dWu, dWd, dwc


def _weights(P, valid, ids, w, slot, norm, reject_policy):
    """Routing weights a [N, k] recomputed from the probabilities P, and the
    combine weights wc after the overflow policy."""
    N, k = ids.shape
    chosen = ids >= 0
    acc = chosen & (slot >= 0)
    m = (np.asarray(w) != 0).astype(np.float64)
    a = np.zeros((N, k))
    s = np.ones(N)
    for t in range(N):
        if not valid[t]:
            continue
        sel = chosen[t]
        pe = P[t, np.where(sel, ids[t], 0)] * sel
        if norm == NORM_FULLPROB:
            a[t] = pe
        else:
            s[t] = pe.sum()
            a[t] = m[t] * pe / s[t] if s[t] > 0 else 0.0
    wc = np.where(acc, a, 0.0)
    rescaled = np.zeros(N, bool)
    A = np.ones(N)
    if reject_policy == 1:
        req = chosen.sum(axis=1)
        rej = (chosen & ~acc).sum(axis=1)
        rescaled = (rej > 0) & (rej < req)
        for t in np.nonzero(rescaled)[0]:
            A[t] = wc[t].sum()
            wc[t] = wc[t] / A[t]
    return a, wc, {"acc": acc, "chosen": chosen, "m": m, "s": s, "A": A, "rescaled": rescaled}


def score_gradient(P, valid, ids, w, slot, dwc, *, norm: int, reject_policy: int = 0, aux_coef: float = 0.0):
    """dL/dg [N, E_r] from the probabilities P [N, E_r] (rows of invalid
    tokens ignored), the routing records and dwc [N, k] = dL/d wc (the
    upstream gradient of each accepted path's combine weight): the chain
    combine weight -> routing weight -> probability -> score of the module
    docstring, plus the balance objective's term."""
    P = np.asarray(P, np.float64)
    ids = np.asarray(ids, np.int64)
    slot = np.asarray(slot, np.int64)
    dwc = np.asarray(dwc, np.float64)
    valid = np.asarray(valid, bool)
    N, E = P.shape
    a, wc, q = _weights(P, valid, ids, w, slot, norm, reject_policy)
    acc, chosen, m, s, A = q["acc"], q["chosen"], q["m"], q["s"], q["A"]
    da = np.where(acc, dwc, 0.0)
    for t in np.nonzero(q["rescaled"])[0]:
        da[t] = np.where(acc[t], (dwc[t] - (dwc[t] * wc[t]).sum()) / A[t], 0.0)
    dG = np.zeros((N, E))
    for t in range(N):
        if not valid[t]:
            continue
        dp = np.zeros(E)
        sel = np.nonzero(chosen[t])[0]
        if norm == NORM_FULLPROB:
            for j in sel:
                dp[ids[t, j]] += da[t, j]
        elif s[t] > 0:
            T = (da[t] * a[t]).sum()
            for j in sel:
                dp[ids[t, j]] += (m[t, j] * da[t, j] - T) / s[t]
        dG[t] = P[t] * (dp - (P[t] * dp).sum())
    if aux_coef != 0.0 and valid.any():
        n = np.bincount(ids[chosen], minlength=E).astype(np.float64)
        if n.sum() > 0:
            f = n / n.sum()
            Pv = P[valid]
            dG[valid] += aux_coef * E / valid.sum() * Pv * (f[None, :] - (Pv @ f)[:, None])
    return dG


def backward(x, W_r, Wg, Wu, Wd, dY, ids, w, slot, *, norm: int, reject_policy: int = 0, b_r=None,
             Ws=None, aux_coef: float = 0.0, bf16=None):
    """Gradients of L (module docstring) for the routing records (ids, w,
    slot) of a forward pass: ids [N, k] chosen experts (-1: pruned or invalid
    token), w [N, k] the forward's routing weights (only their zero pattern is
    read: m_j), slot [N, k] accepted slot (-1: rejected).  Inputs fp32 or bf16
    bit patterns as the forward takes them; dY [N, d] fp32.  bf16 selects the
    precision contract (default: the dtype of x).  Returns a dict of float64
    arrays: dx, dW_r, db_r, dW_g, dW_u, dW_d, dWs_g, dWs_u, dWs_d (None
    without a shared expert), dG (the score gradient [N, E_r]) and dwc
    (dL/d wc per record, 0 where not accepted)."""
    if bf16 is None:
        bf16 = np.asarray(x).dtype == np.uint16
    rnd = bf16_round if bf16 else (lambda v: v)
    X, Wr = _f64(x), _f64(W_r)
    Wg, Wu, Wd = _f64(Wg), _f64(Wu), _f64(Wd)
    N, d = X.shape
    E = Wr.shape[0]
    ids = np.asarray(ids, np.int64)
    slot = np.asarray(slot, np.int64)
    w = np.asarray(w, np.float64)
    k = ids.shape[1] if ids.ndim == 2 else 0
    dYb = rnd(np.asarray(dY, np.float64))

    G = X @ Wr.T
    if b_r is not None:
        G = G + np.asarray(b_r, np.float64)[None, :]
    valid = np.isfinite(G).all(axis=1)
    P = np.zeros((N, E))
    if valid.any():
        Gv = G[valid]
        Pv = np.exp(Gv - Gv.max(axis=1, keepdims=True))
        P[valid] = Pv / Pv.sum(axis=1, keepdims=True)

    a, wc, aux = _weights(P, valid, ids, w, slot, norm, reject_policy)
    acc = aux["acc"]

    dx = np.zeros((N, d))
    dWg, dWu, dWd = np.zeros_like(Wg), np.zeros_like(Wu), np.zeros_like(Wd)
    dwc = np.zeros((N, k))
    for e in range(E):
        tt, jj = np.nonzero(acc & (ids == e))
        if tt.size == 0:
            continue
        order = np.argsort(slot[tt, jj], kind="stable")
        tt, jj = tt[order], jj[order]
        dXe, dWg[e], dWu[e], dWd[e], dwe = _expert_backward(X[tt], Wg[e], Wu[e], Wd[e], dYb[tt], wc[tt, jj],
                                                              rnd, bf16)
        dx[tt] += dXe                      # a token meets an expert at most once
        dwc[tt, jj] = dwe

    out = {"dWs_g": None, "dWs_u": None, "dWs_d": None}
    if Ws is not None and Ws[0] is not None:
        Wsg, Wsu, Wsd = (_f64(a_) for a_ in Ws)
        dXs, out["dWs_g"], out["dWs_u"], out["dWs_d"], _ = _expert_backward(X, Wsg, Wsu, Wsd, dYb, np.ones(N),
                                                                             rnd, bf16)
        dx += dXs

    dG = score_gradient(P, valid, ids, w, slot, dwc, norm=norm, reject_policy=reject_policy, aux_coef=aux_coef)
    dx += dG @ Wr
    out.update({"dx": dx, "dW_r": dG.T @ X, "db_r": dG.sum(axis=0), "dW_g": dWg, "dW_u": dWu, "dW_d": dWd,
                "dG": dG, "dwc": dwc})
    return out


# ---------------------------------------------------------------------------
# Samples of the same gradients, for layers too large to run whole: each is the
# definition above restricted to some hidden units or some tokens (the hidden
# units of an expert are independent of each other, and with aux_coef = 0 a
# token's dx depends on that token's rows only).  Pinned against backward()
# in the CPU tests.
# ---------------------------------------------------------------------------
def expert_backward_columns(X, Wg, Wu, Wd, dY, wc, cols, *, bf16: bool):
    """One expert's weight gradients restricted to hidden units `cols`: rows
    `cols` of dW_g and dW_u and columns `cols` of dW_d, for the expert's
    accepted rows X [R, d] (any order), their upstream rows dY [R, d] (fp32)
    and combine weights wc [R].  Weights as stored (bf16 bit patterns or
    fp32): Wg, Wu [d_f, d], Wd [d, d_f].  Returns float64 (dWg [c, d],
    dWu [c, d], dWd [d, c])."""
    rnd = bf16_round if bf16 else (lambda v: v)
    cols = np.asarray(cols, np.int64)
    X = _f64(X)
    Wg_c, Wu_c = _f64(np.asarray(Wg)[cols]), _f64(np.asarray(Wu)[cols])
    Wd_c = _f64(np.asarray(Wd)[:, cols])
    wc = np.asarray(wc, np.float64)
    dYb = rnd(np.asarray(dY, np.float64))
    Z = X @ Wg_c.T
    U = X @ Wu_c.T
    S, dS = _silu_parts(Z)
    H = S * U
    if bf16:
        H = bf16_round(H)
    dH = wc[:, None] * (dYb @ Wd_c)
    dZ = rnd(dH * U * dS)
    dU = rnd(dH * S)
    dO = rnd(wc[:, None] * dYb)
    return dZ.T @ X, dU.T @ X, dO.T @ H


def token_dx(x, W_r, expert_weights, dY, ids, w, slot, *, norm: int, reject_policy: int = 0, b_r=None,
             bf16: bool):
    """dx of some tokens with aux_coef = 0: x [n, d] their rows, dY [n, d],
    ids / w / slot [n, k] their routing records; expert_weights(e) returns
    (W_g[e], W_u[e], W_d[e]) as stored.  The same chain as backward(): each
    accepted path's expert backward on the token's row, the score gradient
    from its dwc, and dx = sum of the paths' W_g^T dz + W_u^T du + dG W_r.
    Returns float64 [n, d]."""
    rnd = bf16_round if bf16 else (lambda v: v)
    X, Wr = _f64(x), _f64(W_r)
    ids = np.asarray(ids, np.int64)
    slot = np.asarray(slot, np.int64)
    w = np.asarray(w, np.float64)
    n, d = X.shape
    k = ids.shape[1]
    dYb = rnd(np.asarray(dY, np.float64))
    G = X @ Wr.T
    if b_r is not None:
        G = G + np.asarray(b_r, np.float64)[None, :]
    valid = np.isfinite(G).all(axis=1)
    P = np.zeros_like(G)
    if valid.any():
        Gv = G[valid]
        Pv = np.exp(Gv - Gv.max(axis=1, keepdims=True))
        P[valid] = Pv / Pv.sum(axis=1, keepdims=True)
    _, wc, q = _weights(P, valid, ids, w, slot, norm, reject_policy)
    acc = q["acc"]
    dx = np.zeros((n, d))
    dwc = np.zeros((n, k))
    for e in np.unique(ids[acc]):  # each expert's weights converted once, its paths together
        tt, jj = np.nonzero(acc & (ids == e))
        Wg, Wu, Wd = (_f64(a_) for a_ in expert_weights(int(e)))
        dXe, _, _, _, dwe = _expert_backward(X[tt], Wg, Wu, Wd, dYb[tt], wc[tt, jj], rnd, bf16)
        np.add.at(dx, tt, dXe)
        dwc[tt, jj] = dwe
    dG = score_gradient(P, valid, ids, w, slot, dwc, norm=norm, reject_policy=reject_policy, aux_coef=0.0)
    return dx + dG @ Wr


def combine_weights(x, W_r, ids, w, slot, *, norm: int, reject_policy: int = 0, b_r=None):
    """The combine weight wc [n, k] of each accepted path of some tokens (0
    elsewhere), from their rows x [n, d] and routing records: the router's
    probabilities, the routing-weight rule of the layer's normalisation, and
    the overflow policy's rescaling (w is read only for its zero pattern)."""
    X, Wr = _f64(x), _f64(W_r)
    G = X @ Wr.T
    if b_r is not None:
        G = G + np.asarray(b_r, np.float64)[None, :]
    valid = np.isfinite(G).all(axis=1)
    P = np.zeros_like(G)
    if valid.any():
        Gv = G[valid]
        Pv = np.exp(Gv - Gv.max(axis=1, keepdims=True))
        P[valid] = Pv / Pv.sum(axis=1, keepdims=True)
    _, wc, _ = _weights(P, valid, np.asarray(ids, np.int64), np.asarray(w, np.float64), np.asarray(slot, np.int64),
                        norm, reject_policy)
    return wc
