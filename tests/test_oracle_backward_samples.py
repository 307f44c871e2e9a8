"""The sampled gradient functions of the oracle (expert_backward_columns,
token_dx), which the full-size GPU backward tests use, equal the whole-layer
gradient oracle (itself pinned by finite differences and closed forms in
test_oracle_backward_pins.py) on the entries they sample: every weighting
mode, both overflow policies, capacity rejections, fp32 and the bf16
contract."""
import math

import numpy as np
import pytest

import oracle
from seeded_inputs import f32_to_bf16_bits


def _layer(seed, *, N=40, d=16, d_f=12, E=5, k=2, lat=False, bf16=False):
    rng = np.random.default_rng(seed)
    P = {
        "x": rng.standard_normal((N, d)).astype(np.float32),
        "W_r": (rng.standard_normal((E, d)) / math.sqrt(d) * 2).astype(np.float32),
        "b_r": (0.3 * rng.standard_normal(E)).astype(np.float32),
        "W_g": (rng.standard_normal((E, d_f, d)) / math.sqrt(d)).astype(np.float32),
        "W_u": (rng.standard_normal((E, d_f, d)) / math.sqrt(d)).astype(np.float32),
        "W_d": (rng.standard_normal((E, d, d_f)) / math.sqrt(d_f)).astype(np.float32),
    }
    if bf16:
        P = {n: (f32_to_bf16_bits(v) if n != "b_r" else v) for n, v in P.items()}
    lat_v = rng.lognormal(0.0, 0.5, (N, E)).astype(np.float32) if lat else None
    dY = rng.standard_normal((N, d)).astype(np.float32)
    return P, lat_v, dY


CASES = {
    "renorm_capped": dict(k=2, norm=oracle.NORM_RENORM, c=0.75),
    "renorm_policy1_capped_bf16": dict(k=2, norm=oracle.NORM_RENORM, c=0.6, policy=1, bf16=True),
    "fullprob_top1_capped": dict(k=1, norm=oracle.NORM_FULLPROB, c=1.0),
    "wlr": dict(k=3, norm=oracle.NORM_WLR, theta=0.3, lat=True),
    "weight_order_bf16": dict(k=2, norm=oracle.NORM_RENORM, c=0.6, order=1, policy=1, bf16=True),
}


def _run(name):
    cfg = CASES[name]
    P, lat, dY = _layer(31 + len(name), k=cfg["k"], lat=cfg.get("lat", False), bf16=cfg.get("bf16", False))
    out = oracle.forward(P["x"], P["W_r"], P["W_g"], P["W_u"], P["W_d"], k=cfg["k"], norm=cfg["norm"],
                         c=cfg.get("c", 0.0), theta=cfg.get("theta", 0.0), b_r=P["b_r"], lat=lat,
                         reject_policy=cfg.get("policy", 0), accept_order=cfg.get("order", 0))
    if cfg.get("c", 0) > 0:
        assert out["stats"]["rejected"] > 0
    g = oracle.backward(P["x"], P["W_r"], P["W_g"], P["W_u"], P["W_d"], dY, out["ids"], out["w"], out["slot"],
                        norm=cfg["norm"], reject_policy=cfg.get("policy", 0), b_r=P["b_r"], aux_coef=0.0)
    return cfg, P, dY, out, g


@pytest.mark.parametrize("name", list(CASES))
def test_expert_backward_columns_equal_the_whole_layer(name):
    cfg, P, dY, out, g = _run(name)
    ids, slot = np.asarray(out["ids"]), np.asarray(out["slot"])
    bf16 = bool(cfg.get("bf16", False))
    wc_all = oracle.combine_weights(P["x"], P["W_r"], ids, out["w"], slot, norm=cfg["norm"],
                                    reject_policy=cfg.get("policy", 0), b_r=P["b_r"])
    E = np.asarray(P["W_g"]).shape[0]
    d_f = np.asarray(P["W_g"]).shape[1]
    checked = 0
    for e in range(E):
        tt, jj = np.nonzero((ids == e) & (slot >= 0))
        if tt.size == 0:
            continue
        wc = wc_all[tt, jj]
        cols = np.array([0, d_f // 2, d_f - 1])
        dWg, dWu, dWd = oracle.expert_backward_columns(P["x"][tt], P["W_g"][e], P["W_u"][e], P["W_d"][e], dY[tt],
                                                       wc, cols, bf16=bf16)
        np.testing.assert_allclose(dWg, g["dW_g"][e][cols], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dWu, g["dW_u"][e][cols], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dWd, g["dW_d"][e][:, cols], rtol=1e-12, atol=1e-12)
        checked += 1
    assert checked >= 3


@pytest.mark.parametrize("name", list(CASES))
def test_token_dx_equals_the_whole_layer(name):
    cfg, P, dY, out, g = _run(name)
    rows = np.array([0, 3, 7, 11, 20, 39])
    ids, w, slot = (np.asarray(out[n])[rows] for n in ("ids", "w", "slot"))
    dx = oracle.token_dx(P["x"][rows], P["W_r"], lambda e: (P["W_g"][e], P["W_u"][e], P["W_d"][e]), dY[rows],
                         ids, w, slot, norm=cfg["norm"], reject_policy=cfg.get("policy", 0), b_r=P["b_r"],
                         bf16=bool(cfg.get("bf16", False)))
    np.testing.assert_allclose(dx, g["dx"][rows], rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("name", list(CASES))
def test_combine_weights_are_the_forwards(name):
    """The combine weights recomputed from the rows equal the forward oracle's
    routing weights on accepted paths (with policy 1's rescaling of a token
    that lost some but not all of its paths)."""
    cfg, P, dY, out, g = _run(name)
    ids, slot, w = np.asarray(out["ids"]), np.asarray(out["slot"]), np.asarray(out["w"], np.float64)
    wc = oracle.combine_weights(P["x"], P["W_r"], ids, w, slot, norm=cfg["norm"], reject_policy=cfg.get("policy", 0),
                                b_r=P["b_r"])
    acc = (ids >= 0) & (slot >= 0)
    want = np.where(acc, w, 0.0)
    if cfg.get("policy", 0) == 1:
        req = (ids >= 0).sum(axis=1)
        rej = ((ids >= 0) & ~acc).sum(axis=1)
        part = (rej > 0) & (rej < req)
        want[part] = want[part] / want[part].sum(axis=1, keepdims=True)
    np.testing.assert_allclose(wc, want, rtol=1e-6, atol=1e-7)
