"""The gradient oracle against automatic differentiation of an independent
restatement of the layer.

The forward is written out again here with torch operations in float64 on the
CPU ("LLM from scratch" ch. 36.1-36.4: scores, softmax, the weighting of the
chosen experts, the overflow policy, the combine Y_t = sum wc_j E_e(x_t), the
shared expert, the balance objective E_r sum_e f_e pbar_e with the shares f
held constant), with the routing decisions (ids, slot) taken from the forward
oracle.  torch's reverse-mode differentiation of that function is a library
routine independent of oracle/backward.py; every coordinate of every
gradient must agree to rounding (1e-10 relative to the largest entry).
"""
import math

import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")


def _case(seed, N, d, d_f, E, shared):
    rng = np.random.default_rng(seed)
    P = {
        "x": rng.standard_normal((N, d)).astype(np.float32),
        "W_r": (rng.standard_normal((E, d)) / math.sqrt(d) * 2).astype(np.float32),
        "b_r": (0.3 * rng.standard_normal(E)).astype(np.float32),
        "W_g": (rng.standard_normal((E, d_f, d)) / math.sqrt(d)).astype(np.float32),
        "W_u": (rng.standard_normal((E, d_f, d)) / math.sqrt(d)).astype(np.float32),
        "W_d": (rng.standard_normal((E, d, d_f)) / math.sqrt(d_f)).astype(np.float32),
    }
    if shared:
        P["Ws_g"] = (rng.standard_normal((shared, d)) / math.sqrt(d)).astype(np.float32)
        P["Ws_u"] = (rng.standard_normal((shared, d)) / math.sqrt(d)).astype(np.float32)
        P["Ws_d"] = (rng.standard_normal((d, shared)) / math.sqrt(shared)).astype(np.float32)
    lat = rng.lognormal(0.0, 0.5, (N, E)).astype(np.float32)
    dY = rng.standard_normal((N, d))
    return P, lat, dY


def _swiglu(x, Wg, Wu, Wd):
    z = x @ Wg.T
    return (z * torch.sigmoid(z) * (x @ Wu.T)) @ Wd.T


def _loss(T, ids, slot, w, dY, norm, policy, lam):
    """<dY, Y> + lam * aux, written out per token with the decisions fixed."""
    x, W_r = T["x"], T["W_r"]
    G = x @ W_r.T + T["b_r"]
    P = torch.softmax(G, dim=1)
    N, k = ids.shape
    E = W_r.shape[0]
    rows = []
    for t in range(N):
        sel = [j for j in range(k) if ids[t, j] >= 0]
        y = torch.zeros(x.shape[1], dtype=x.dtype)
        if sel:
            pe = torch.stack([P[t, ids[t, j]] for j in sel])
            if norm == oracle.NORM_FULLPROB:
                a = pe
            else:
                m = torch.tensor([1.0 if w[t, j] != 0 else 0.0 for j in sel], dtype=x.dtype)
                a = m * pe / pe.sum()
            acc = [slot[t, j] >= 0 for j in sel]
            wc = a * torch.tensor([1.0 if s else 0.0 for s in acc], dtype=x.dtype)
            if policy == 1 and 0 < sum(not s for s in acc) < len(sel):
                wc = wc / wc.sum()
            for i, j in enumerate(sel):
                if acc[i]:
                    e = ids[t, j]
                    y = y + wc[i] * _swiglu(x[t:t + 1], T["W_g"][e], T["W_u"][e], T["W_d"][e])[0]
        rows.append(y)
    Y = torch.stack(rows)
    if "Ws_g" in T:
        Y = Y + _swiglu(x, T["Ws_g"], T["Ws_u"], T["Ws_d"])
    L = (torch.from_numpy(dY) * Y).sum()
    if lam:
        n = np.bincount(ids[ids >= 0], minlength=E).astype(np.float64)
        f = torch.from_numpy(n / n.sum())
        L = L + lam * E * (f * P.mean(dim=0)).sum()
    return L


@pytest.mark.parametrize("norm,k,c,policy,order,lam,shared", [
    (oracle.NORM_RENORM, 2, 0.75, 0, 0, 0.7, 0),
    (oracle.NORM_RENORM, 2, 0.75, 1, 0, 0.0, 5),
    (oracle.NORM_FULLPROB, 1, 1.0, 0, 0, 0.5, 0),
    (oracle.NORM_WLR, 3, 0.0, 0, 0, 0.2, 0),
    (oracle.NORM_RENORM, 2, 0.6, 1, 1, 0.3, 4),
    (oracle.NORM_FULLPROB, 4, 0.5, 1, 1, 1.0, 0),
])
def test_gradients_equal_automatic_differentiation(norm, k, c, policy, order, lam, shared):
    N, d, d_f, E = 24, 12, 6, 4
    P, lat, dY = _case(40 + k + 3 * policy + 5 * order, N, d, d_f, E, shared)
    Ws = (P["Ws_g"], P["Ws_u"], P["Ws_d"]) if shared else None
    out = oracle.forward(P["x"], P["W_r"], P["W_g"], P["W_u"], P["W_d"], k=k, norm=norm, c=c, theta=0.3,
                         b_r=P["b_r"], lat=lat if norm == oracle.NORM_WLR else None, Ws=Ws,
                         reject_policy=policy, accept_order=order)
    if c > 0:
        assert out["stats"]["rejected"] > 0
    g = oracle.backward(P["x"], P["W_r"], P["W_g"], P["W_u"], P["W_d"], dY, out["ids"], out["w"], out["slot"],
                        norm=norm, reject_policy=policy, b_r=P["b_r"], Ws=Ws, aux_coef=lam)
    T = {n: torch.tensor(a.astype(np.float64), requires_grad=True) for n, a in P.items()}
    L = _loss(T, out["ids"], out["slot"], out["w"], dY, norm, policy, lam)
    L.backward()
    names = {"x": "dx", "W_r": "dW_r", "b_r": "db_r", "W_g": "dW_g", "W_u": "dW_u", "W_d": "dW_d",
             "Ws_g": "dWs_g", "Ws_u": "dWs_u", "Ws_d": "dWs_d"}
    for n, t in T.items():
        ref = t.grad.numpy()
        got = g[names[n]]
        scale = max(np.abs(ref).max(), 1e-300)
        assert np.abs(got - ref).max() <= 1e-10 * scale, (n, np.abs(got - ref).max() / scale)
