"""Pins of the gradient oracle (oracle/backward.py) against things other than
itself:

- central finite differences of the forward oracle (pinned on its own in
  test_oracle_pins.py) and of the balance objective's value, on tiny fp32
  layers in every weighting mode, overflow policy and acceptance order, with
  and without a shared expert;
- closed forms on the worked example of "LLM from scratch" ch. 36.4 (N = 4,
  E_r = 3, k = 2, the page's linear experts F_e(x) = e x): the score gradient
  of each token's output, with the capacity rejection and both overflow
  policies;
- the balance objective's stationary point (uniform shares and
  probabilities) and the page's remark that its gradient reaches experts that
  were not chosen;
- the bf16 rounding against the library's conversion, and the bf16 contract
  within bf16 error of the exact gradient.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from seeded_inputs import f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(seed, *, N=20, d=12, d_f=6, E=4, k=2, shared=0, lat=False, bias=True):
    rng = np.random.default_rng(seed)
    P = {
        "x": rng.standard_normal((N, d)).astype(np.float32),
        "W_r": (rng.standard_normal((E, d)) / math.sqrt(d) * 2).astype(np.float32),
        "W_g": (rng.standard_normal((E, d_f, d)) / math.sqrt(d)).astype(np.float32),
        "W_u": (rng.standard_normal((E, d_f, d)) / math.sqrt(d)).astype(np.float32),
        "W_d": (rng.standard_normal((E, d, d_f)) / math.sqrt(d_f)).astype(np.float32),
    }
    if bias:
        P["b_r"] = (0.3 * rng.standard_normal(E)).astype(np.float32)
    if shared:
        P["Ws_g"] = (rng.standard_normal((shared, d)) / math.sqrt(d)).astype(np.float32)
        P["Ws_u"] = (rng.standard_normal((shared, d)) / math.sqrt(d)).astype(np.float32)
        P["Ws_d"] = (rng.standard_normal((d, shared)) / math.sqrt(shared)).astype(np.float32)
    extra = {"lat": rng.lognormal(0.0, 0.5, (N, E)).astype(np.float32) if lat else None,
             "dY": rng.standard_normal((N, d)).astype(np.float32)}
    return P, extra


def _forward(P, extra, cfg):
    Ws = (P["Ws_g"], P["Ws_u"], P["Ws_d"]) if "Ws_g" in P else None
    return oracle.forward(P["x"], P["W_r"], P["W_g"], P["W_u"], P["W_d"], k=cfg["k"], norm=cfg["norm"],
                          c=cfg.get("c", 0.0), theta=cfg.get("theta", 0.0), b_r=P.get("b_r"), lat=extra["lat"],
                          Ws=Ws, reject_policy=cfg.get("policy", 0), accept_order=cfg.get("order", 0))


def _loss(P, extra, cfg):
    out = _forward(P, extra, cfg)
    val = float((extra["dY"].astype(np.float64) * out["Y"]).sum())
    lam = cfg.get("aux", 0.0)
    if lam:
        r = oracle.route(P["x"], P["W_r"], k=cfg["k"], norm=cfg["norm"], theta=cfg.get("theta", 0.0),
                         b_r=P.get("b_r"), lat=extra["lat"])
        val += lam * oracle.aux_balance(r["logits"], out["ids"], P["W_r"].shape[0])
    return val, out["ids"], out["slot"]


CASES = {
    "renorm_capped_aux": dict(k=2, norm=oracle.NORM_RENORM, c=0.75, aux=0.7),
    "renorm_policy1_shared": dict(k=2, norm=oracle.NORM_RENORM, c=0.75, policy=1, shared=5),
    "switch_fullprob_aux": dict(k=1, norm=oracle.NORM_FULLPROB, c=1.0, aux=0.5),
    "wlr_theta": dict(k=3, norm=oracle.NORM_WLR, theta=0.3, lat=True),
    "weight_order_capped": dict(k=2, norm=oracle.NORM_RENORM, c=0.6, order=1, policy=1, aux=0.2),
    "k3_uncapped_shared": dict(k=3, norm=oracle.NORM_RENORM, shared=4),
}

GRAD_OF = {"x": "dx", "W_r": "dW_r", "b_r": "db_r", "W_g": "dW_g", "W_u": "dW_u", "W_d": "dW_d",
           "Ws_g": "dWs_g", "Ws_u": "dWs_u", "Ws_d": "dWs_d"}


@pytest.mark.parametrize("name", list(CASES))
def test_gradients_equal_finite_differences_of_the_forward(name):
    cfg = CASES[name]
    P, extra = _case(11 + len(name), k=cfg["k"], shared=cfg.get("shared", 0), lat=cfg.get("lat", False))
    out = _forward(P, extra, cfg)
    if cfg.get("c", 0) > 0:
        assert out["stats"]["rejected"] > 0          # the capacity binds: rejection paths are exercised
    Ws = (P["Ws_g"], P["Ws_u"], P["Ws_d"]) if "Ws_g" in P else None
    g = oracle.backward(P["x"], P["W_r"], P["W_g"], P["W_u"], P["W_d"], extra["dY"], out["ids"], out["w"],
                        out["slot"], norm=cfg["norm"], reject_policy=cfg.get("policy", 0), b_r=P.get("b_r"),
                        Ws=Ws, aux_coef=cfg.get("aux", 0.0))
    base_ids, base_slot = out["ids"], out["slot"]
    rng = np.random.default_rng(5)
    h = 2.0 ** -10
    checked = 0
    for pname in P:
        grad = g[GRAD_OF[pname]]
        arr = P[pname]
        scale = 1.0 + np.abs(grad).max()
        for idx in rng.choice(arr.size, size=min(6, arr.size), replace=False):
            orig = arr.flat[idx]
            hi, lo = np.float32(orig + h), np.float32(orig - h)
            arr.flat[idx] = hi
            Lp, ip, sp = _loss(P, extra, cfg)
            arr.flat[idx] = lo
            Lm, im, sm = _loss(P, extra, cfg)
            arr.flat[idx] = orig
            if not (np.array_equal(ip, base_ids) and np.array_equal(im, base_ids) and
                    np.array_equal(sp, base_slot) and np.array_equal(sm, base_slot)):
                continue                               # a routing decision moved: not differentiable here
            fd = (Lp - Lm) / (float(hi) - float(lo))
            assert abs(fd - grad.flat[idx]) <= 2e-6 * scale, (pname, int(idx), fd, grad.flat[idx])
            checked += 1
    assert checked >= 5 * len(P)


def test_gradient_is_linear_in_the_upstream_gradient():
    cfg = CASES["renorm_policy1_shared"]
    P, extra = _case(3, shared=5)
    out = _forward(P, extra, cfg)
    Ws = (P["Ws_g"], P["Ws_u"], P["Ws_d"])
    rng = np.random.default_rng(9)
    dY1 = rng.standard_normal(extra["dY"].shape)
    dY2 = rng.standard_normal(extra["dY"].shape)

    def run(dY):
        return oracle.backward(P["x"], P["W_r"], P["W_g"], P["W_u"], P["W_d"], dY, out["ids"], out["w"],
                               out["slot"], norm=cfg["norm"], reject_policy=1, b_r=P["b_r"], Ws=Ws)
    g1, g2, g12 = run(dY1), run(dY2), run(dY1 + 2.0 * dY2)
    for key in ("dx", "dW_r", "db_r", "dW_g", "dW_u", "dW_d", "dWs_g", "dWs_u", "dWs_d"):
        np.testing.assert_allclose(g12[key], g1[key] + 2.0 * g2[key], rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------
# the worked example of ch. 36.4 with the page's linear experts
# ---------------------------------------------------------------------------
def _n4():
    g = json.load(open(os.path.join(GOLDEN, "n4_e3_k2_example.json")))
    P = np.array(g["probabilities"], np.float64)          # [token, expert], rows sum to one
    return P


def _example_score_gradient(policy, C):
    """Score gradient of L = sum_t <x_t, Y_t> on the example (X = I_4, so
    dY_t = x_t), where expert e (1-based) is F_e(x) = e x: the upstream
    gradient of a path's combine weight is <x_t, e x_t> = e."""
    P = _n4()
    ids = np.argsort(-P, axis=1, kind="stable")[:, :2]
    w = P[np.arange(4)[:, None], ids] / P[np.arange(4)[:, None], ids].sum(axis=1, keepdims=True)
    d = oracle.dispatch(ids.astype(np.int32), E=3, C=C)
    dwc = (ids + 1).astype(np.float64) * (d["slot"] >= 0)
    return oracle.score_gradient(P, np.ones(4, bool), ids, w, d["slot"], dwc, norm=oracle.NORM_RENORM,
                                 reject_policy=policy)


def test_example_score_gradient_uncapped_closed_form():
    # token t chooses experts (i, j) with i < j; Y_t = (i p_i + j p_j)/(p_i + p_j) x_t,
    # so <x_t, Y_t> = i + (j - i) sigma(g_j - g_i) and its score gradient is
    # (j - i) sigma (1 - sigma) on g_j, the negative on g_i, 0 on the third.
    # Probabilities of the page's table: sigma = 2/9, 1/3, 7/18, 7/9.
    dG = _example_score_gradient(0, C=4)
    q = [Fraction(2, 9), Fraction(1, 3), Fraction(7, 18), Fraction(7, 9)]
    pairs = [(0, 1), (0, 1), (0, 1), (1, 2)]
    for t, ((i, j), s) in enumerate(zip(pairs, q)):
        want = np.zeros(3)
        v = float((j - i) * s * (1 - s))
        want[j], want[i] = v, -v
        np.testing.assert_allclose(dG[t], want, rtol=0, atol=1e-15)
    # values as fractions: 14/81, 2/9, 77/324, 14/81
    assert abs(dG[0, 1] - 14 / 81) < 1e-15 and abs(dG[2, 1] - 77 / 324) < 1e-15


def test_example_score_gradient_with_the_rejection_both_policies():
    # C = 3 (gamma = 1): expert 2 rejects token 4 (token order).  Policy 0:
    # Y_4 = 3 a_3 x_4 = 3 sigma(g_3 - g_2) x_4, gradient 3 sigma (1 - sigma) =
    # 14/27 on g_3 and -14/27 on g_2.  Policy 1 (remaining path renormalised):
    # Y_4 = 3 x_4 whatever the scores, gradient 0.  Tokens 1-3 are unchanged.
    g0 = _example_score_gradient(0, C=3)
    g1 = _example_score_gradient(1, C=3)
    full = _example_score_gradient(0, C=4)
    np.testing.assert_allclose(g0[3], [0.0, -14 / 27, 14 / 27], rtol=0, atol=1e-15)
    np.testing.assert_allclose(g1[3], [0.0, 0.0, 0.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(g0[:3], full[:3], rtol=0, atol=0)
    np.testing.assert_allclose(g1[:3], full[:3], rtol=0, atol=0)


def test_balance_objective_gradient_on_the_example_equals_finite_differences():
    # the objective's value on the example is pinned to 1.0359375 elsewhere;
    # its score gradient here against central differences of that value with
    # the chosen sets held fixed.  It is nonzero on unchosen experts (the page:
    # the objective trains scores that were not selected).
    P = _n4()
    G = np.log(P)
    ids = np.argsort(-P, axis=1, kind="stable")[:, :2]
    dG = oracle.score_gradient(P, np.ones(4, bool), ids, np.ones((4, 2)), np.zeros((4, 2), np.int32),
                               np.zeros((4, 2)), norm=oracle.NORM_RENORM, aux_coef=1.0)
    h = 1e-6
    for t in range(4):
        for e in range(3):
            Gp, Gm = G.copy(), G.copy()
            Gp[t, e] += h
            Gm[t, e] -= h
            fd = (oracle.aux_balance(Gp, ids, 3) - oracle.aux_balance(Gm, ids, 3)) / (2 * h)
            assert abs(fd - dG[t, e]) < 1e-8, (t, e, fd, dG[t, e])
    unchosen = np.ones((4, 3), bool)
    unchosen[np.arange(4)[:, None], ids] = False
    assert (np.abs(dG[unchosen]) > 1e-3).all()


def test_balance_objective_uniform_point_is_stationary():
    # f_e = pbar_e = 1/E_r: every score gradient vanishes (f_e - sum_i f_i p_i = 0)
    E = 4
    P = np.full((8, E), 1.0 / E)
    ids = np.array([[e] for e in range(E)] * 2)
    dG = oracle.score_gradient(P, np.ones(8, bool), ids, np.ones((8, 1)), np.zeros((8, 1), np.int32),
                               np.zeros((8, 1)), norm=oracle.NORM_FULLPROB, aux_coef=1.0)
    assert np.abs(dG).max() < 1e-16


# ---------------------------------------------------------------------------
# bf16
# ---------------------------------------------------------------------------
def test_bf16_round_matches_the_library_conversion():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        1.0 + np.arange(-64, 64) * 2.0 ** -9,          # ties at 1 + odd 2^-8 multiples
                        [0.0, -0.0, 2.0 ** -130, 3.0 * 2.0 ** -133, 65504.0]]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_round(v.astype(np.float64))
    np.testing.assert_array_equal(got, want)
    for val in v[:200]:
        assert oracle.round_bf16(float(val)) == oracle.bf16_round(float(val))


def test_bf16_contract_within_bf16_error_of_the_exact_gradient():
    cfg = CASES["renorm_policy1_shared"]
    P, extra = _case(21, d=16, d_f=8, shared=8)
    Pb = {n: f32_to_bf16_bits(a) if n != "b_r" else a for n, a in P.items()}
    out = oracle.forward(Pb["x"], Pb["W_r"], Pb["W_g"], Pb["W_u"], Pb["W_d"], k=2, norm=cfg["norm"], c=0.75,
                         b_r=P["b_r"], Ws=(Pb["Ws_g"], Pb["Ws_u"], Pb["Ws_d"]), reject_policy=1)
    args = (Pb["x"], Pb["W_r"], Pb["W_g"], Pb["W_u"], Pb["W_d"], extra["dY"], out["ids"], out["w"], out["slot"])
    kw = dict(norm=cfg["norm"], reject_policy=1, b_r=P["b_r"], Ws=(Pb["Ws_g"], Pb["Ws_u"], Pb["Ws_d"]))
    gb = oracle.backward(*args, **kw)                 # bf16 contract (inputs are bf16)
    ge = oracle.backward(*args, bf16=False, **kw)     # exact arithmetic on the same bf16 values
    for key in ("dx", "dW_r", "dW_g", "dW_u", "dW_d", "dWs_g", "dWs_u", "dWs_d"):
        rel = np.linalg.norm(gb[key] - ge[key]) / np.linalg.norm(ge[key])
        assert 0 < rel < 2e-2, (key, rel)
