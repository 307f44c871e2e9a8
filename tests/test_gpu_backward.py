"""Backward pass on the GPU (moe_backward through the C ABI) against the
gradient oracle, on seeded inputs.

The oracle runs on the GPU forward's own routing records (ids, weights,
slots), so both sides differentiate the same piecewise-smooth function.
Tolerances (max-abs error over max-abs reference, per gradient):
  * expert and shared-expert weight gradients and dx: 5e-3.  The tensor-core
    operands (dY, wc dY, dz, du and the forward's h) are bf16 on both sides,
    but the GPU rounds values it accumulated in fp32, so an operand can land
    one bf16 step (2^-8 = 3.9e-3 relative) away from the oracle's where the
    fp32 value sits near a rounding boundary; such a flip moves one term of
    a sum, so an output element moves by less than 2^-8 of the largest
    output, plus fp32 accumulation error;
  * router gradients dW_r and db_r: 2e-3.  They come from the combine-weight
    gradients <W_d^T dY_t, h>, fp32 sums over d_f of bf16-exact products,
    and fp32 router arithmetic; a missing term of the chain (an overflow
    policy, the renormalisation, the balance objective) moves them by far
    more;
  * the balance objective's gradient alone (dY = 0): 1e-4.
  * fp32 layers (CUDA-core contractions, nothing rounded): 1e-4, the forward's
    fp32 bound.
Cases span single-CTA and CTA-pair tiles, ragged row, column and K tails,
capacity rejection under both overflow policies, acceptance by weight, WLR
pruning, a shared expert, an expert count that is not a multiple of 4 (score
recomputation on the CUDA cores), fp32 layers and the empty batch.
"""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - GPU tests need a device
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_25_b200 as moe  # noqa: E402

W = si.WORKLOADS
CASES = {
    "mixtral_small": W["mixtral_bf16"].scaled("bwd_mixtral_small", N=512, d=320, d_f=384),
    "pair_tiles": W["mixtral_bf16"].scaled("bwd_pair", N=1600, d=320, d_f=384, E=2, k=1),
    # d_f = 800 >= 768: dW_g and dW_u run on CTA pairs (and d = 192: dW_d on
    # single CTAs), both with the weight-gradient epilogue and ragged tiles
    "pair_weight_grads": W["mixtral_bf16"].scaled("bwd_pair_dw", N=300, d=192, d_f=800, E=4, k=2),
    "qwen3_capped_aux": W["qwen3_skew_bf16"].scaled("bwd_qwen3", N=1024, d=256, d_f=192, E=32, k=4),
    "deepseek_shared": W["deepseek_shared_bf16"].scaled("bwd_deepseek", N=384, d=448, d_f=128, E=64, k=6,
                                                        d_f_shared=192),
    "wdmoe_wlr": W["wdmoe_decode_bf16"].scaled("bwd_wdmoe", N=64, d=512, d_f=640),
    "renorm_reject": W["qwen3_skew_bf16"].scaled("bwd_renorm_reject", N=1024, d=256, d_f=192, E=16, k=2,
                                                 reject_policy=1),
    "weight_order": W["qwen3_skew_bf16"].scaled("bwd_weight_order", N=700, d=128, d_f=192, E=16, k=2, c=0.8,
                                                accept_order=1, reject_policy=1),
    "odd_experts": W["mixtral_bf16"].scaled("bwd_odd_experts", N=200, d=64, d_f=64, E=34, k=3, c=1.0),
    # 128 experts: router contractions on the tensor cores (bf16 hi + lo parts of
    # the score gradient), N not a multiple of 32, K split over the tokens for dW_r
    "wide_router_aux": W["qwen3_skew_bf16"].scaled("bwd_wide_router", N=520, d=192, d_f=128, E=128, k=8),
    "one_expert_ragged": W["mixtral_bf16"].scaled("bwd_one_expert", N=200, d=64, d_f=136, E=1, k=1),
    # fp32 layers (every contraction on the CUDA cores, nothing rounded)
    "switch_f32_capped": W["switch_top1_f32"].scaled("bwd_switch_f32", N=1000, d=72, d_f=96, c=0.9),
    "renorm_f32_shared_policy1": W["switch_top1_f32"].scaled("bwd_f32_shared", N=500, d=64, d_f=80, E=6, k=2,
                                                            norm=si.NORM_RENORM, c=0.8, d_f_shared=40,
                                                            reject_policy=1),
}
AUX = {"qwen3_capped_aux": 0.5, "weight_order": 0.3, "odd_experts": 1.0, "switch_f32_capped": 0.5,
       "wide_router_aux": 0.5}


def _grads(w, device="cuda"):
    shapes = {"dx": (w.N, w.d), "dW_r": (w.E, w.d), "db_r": (w.E,), "dW_g": (w.E, w.d_f, w.d),
              "dW_u": (w.E, w.d_f, w.d), "dW_d": (w.E, w.d, w.d_f)}
    if w.d_f_shared:
        shapes.update({"dWs_g": (w.d_f_shared, w.d), "dWs_u": (w.d_f_shared, w.d), "dWs_d": (w.d, w.d_f_shared)})
    return {n: torch.full(s, float("nan"), dtype=torch.float32, device=device) for n, s in shapes.items()}


def _backward(w, inp, full, dY, aux):
    p, dev, ws = full["p"], full["dev"], full["ws"]
    g = _grads(w)
    bws = torch.empty(moe.moe_backward_workspace_size(p, full["rec"]["offsets"] if w.N else None),
                      dtype=torch.uint8, device="cuda")
    moe.moe_backward(p, full["rec"]["offsets"], dev["x"], dev["W_r"], dev.get("b_r"), dev["W_g"], dev["W_u"],
                     dev["W_d"], dev.get("Ws_g"), dev.get("Ws_u"), dev.get("Ws_d"),
                     torch.from_numpy(dY).cuda(), ws, g, bws, aux_coef=aux)
    assert moe.moe_backward_check(p, bws) == moe.MOE_OK
    return {n: t.cpu().numpy().astype(np.float64) for n, t in g.items()}


def _reference(w, inp, rec, dY, aux):
    Ws = (inp["Ws_g"], inp["Ws_u"], inp["Ws_d"]) if w.d_f_shared else None
    return oracle.backward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], dY, rec["ids"], rec["w"],
                           rec["slot"], norm=w.norm, reject_policy=w.reject_policy, b_r=inp.get("b_r"), Ws=Ws,
                           aux_coef=aux)


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    w = CASES[name]
    inp = si.inputs(w)
    full = parity.gpu_forward(w, inp)
    assert full["status"] == moe.MOE_OK
    if w.c > 0:
        assert full["stats"]["rejected"] > 0       # the capacity binds
    dY = si.upstream_gradient(w)
    aux = AUX.get(name, 0.0)
    got = _backward(w, inp, full, dY, aux)
    ref = _reference(w, inp, full["rec"], dY, aux)
    errs = {}
    for n, g in got.items():
        assert np.isfinite(g).all(), n
        errs[n] = parity.rel_err(g, ref[n])
        tol = 2e-3 if n in ("dW_r", "db_r") else 5e-3
        if w.dtype == si.DT_F32:
            tol = 1e-4       # fp32 accumulation against float64, nothing rounded
        assert errs[n] <= tol, (n, errs[n], errs)
    # experts that received no rows have exactly zero weight gradients
    empty = np.nonzero(full["rec"]["acc"] == 0)[0]
    for e in empty:
        assert not got["dW_g"][e].any() and not got["dW_u"][e].any() and not got["dW_d"][e].any()


def test_balance_objective_gradient_alone():
    w = CASES["qwen3_capped_aux"]
    inp = si.inputs(w)
    full = parity.gpu_forward(w, inp)
    dY = np.zeros((w.N, w.d), np.float32)
    got = _backward(w, inp, full, dY, 1.0)
    ref = _reference(w, inp, full["rec"], dY, 1.0)
    for n in ("dW_g", "dW_u", "dW_d"):
        assert not got[n].any(), n
    for n in ("dx", "dW_r", "db_r"):
        assert np.abs(ref[n]).max() > 0
        assert parity.rel_err(got[n], ref[n]) <= 1e-4, n


def test_backward_empty_batch():
    w = CASES["mixtral_small"].scaled("bwd_empty", N=0)
    inp = si.inputs(w)
    full = parity.gpu_forward(w, inp)
    got = _backward(w, inp, full, np.zeros((0, w.d), np.float32), 0.0)
    for n, g in got.items():
        assert not g.any(), n


def test_backward_rejects_bad_offsets():
    w = CASES["mixtral_small"]
    inp = si.inputs(w)
    full = parity.gpu_forward(w, inp)
    p, dev = full["p"], full["dev"]
    g = _grads(w)
    bws = torch.empty(moe.moe_backward_workspace_size(p), dtype=torch.uint8, device="cuda")
    bad = full["rec"]["offsets"].copy()
    bad[-1] = w.N * w.k + 1
    dY = torch.zeros(w.N, w.d, device="cuda")
    with pytest.raises(moe.MoEError):
        moe.moe_backward(p, bad, dev["x"], dev["W_r"], None, dev["W_g"], dev["W_u"], dev["W_d"], None, None, None,
                         dY, full["ws"], g, bws)


def test_backward_check_reports_stale_host_offsets():
    """Host offsets that pass the host checks (a non-decreasing prefix from 0)
    but are not the forward's: the backward sizes its launches from them, so
    moe_backward_check must report the mismatch instead of MOE_OK."""
    w = CASES["mixtral_small"]
    inp = si.inputs(w)
    full = parity.gpu_forward(w, inp)
    p, dev = full["p"], full["dev"]
    g = _grads(w)
    good = full["rec"]["offsets"].astype(np.int32)
    stale = (good // 2).astype(np.int32)          # every expert with about half its rows
    assert (np.diff(stale) >= 0).all() and stale[0] == 0 and (stale != good).any()
    dY = torch.zeros(w.N, w.d, device="cuda")
    for offs, want in ((stale, moe.MOE_ERR_INVALID_ARG), (good, moe.MOE_OK)):
        bws = torch.empty(moe.moe_backward_workspace_size(p, offs), dtype=torch.uint8, device="cuda")
        moe.moe_backward(p, offs, dev["x"], dev["W_r"], None, dev["W_g"], dev["W_u"], dev["W_d"], None, None, None,
                         dY, full["ws"], g, bws)
        assert moe.moe_backward_check(p, bws) == want


@pytest.mark.parametrize("name", ["mixtral_bf16", "qwen3_skew_bf16"])
def test_full_size_backward_sampled(name):
    """The backward of the page-shaped layers at full size, in the benchmark's
    launch configuration (CTA-pair weight gradients on the Mixtral shape, the
    tensor-core router contractions on the Qwen3 shape), checked on samples the
    oracle computes one by one: rows of dW_g and dW_u and columns of dW_d for
    six hidden units of three experts (the most loaded, a middle one and the
    least loaded), and dx of 16 tokens (every path, including rejected ones).
    Each sampled row within the bf16 bound on its own; aux_coef = 0, so a
    token's dx depends on its own rows only."""
    w = si.WORKLOADS[name]
    inp = si.inputs(w)
    full = parity.gpu_forward(w, inp)
    assert full["status"] == moe.MOE_OK
    rec = full["rec"]
    p, dev, ws = full["p"], full["dev"], full["ws"]
    dY = si.upstream_gradient(w)
    g = _grads(w)
    bws = torch.empty(moe.moe_backward_workspace_size(p, rec["offsets"]), dtype=torch.uint8, device="cuda")
    moe.moe_backward(p, rec["offsets"], dev["x"], dev["W_r"], dev.get("b_r"), dev["W_g"], dev["W_u"], dev["W_d"],
                     None, None, None, torch.from_numpy(dY).cuda(), ws, g, bws, aux_coef=0.0)
    assert moe.moe_backward_check(p, bws) == moe.MOE_OK
    ids, wts, slot = rec["ids"], rec["w"], rec["slot"]
    acc_rows = np.array([int(((ids == e) & (slot >= 0)).sum()) for e in range(w.E)])
    live = np.nonzero(acc_rows > 0)[0]
    order = live[np.argsort(acc_rows[live], kind="stable")]
    experts = [int(order[-1]), int(order[len(order) // 2]), int(order[0])]
    rng = np.random.default_rng(17)
    cols = np.unique(np.concatenate([[0, w.d_f // 3, 2 * w.d_f // 3, w.d_f - 1], rng.integers(0, w.d_f, 2)]))
    wc = oracle.combine_weights(inp["x"], inp["W_r"], ids, wts, slot, norm=w.norm, reject_policy=w.reject_policy,
                                b_r=inp.get("b_r"))
    cols_t = torch.from_numpy(cols).cuda()
    worst = {}
    for e in experts:
        tt, jj = np.nonzero((ids == e) & (slot >= 0))
        ref = oracle.expert_backward_columns(inp["x"][tt], inp["W_g"][e], inp["W_u"][e], inp["W_d"][e], dY[tt],
                                             wc[tt, jj], cols, bf16=True)
        got = (g["dW_g"][e].index_select(0, cols_t), g["dW_u"][e].index_select(0, cols_t),
               g["dW_d"][e].index_select(1, cols_t).T)
        for n, r_, g_ in zip(("dW_g", "dW_u", "dW_d"), (ref[0], ref[1], ref[2].T), got):
            g_ = g_.cpu().numpy().astype(np.float64)
            assert np.isfinite(g_).all()
            err, row = parity.rel_err(g_, r_), parity.row_rel_err(g_, r_)
            worst[n] = max(worst.get(n, 0.0), row)
            assert err <= 5e-3 and row <= 1e-2, (name, n, e, err, row)
    # tokens: seeded, plus (when the capacity binds) tokens that lost a path
    lost = np.nonzero(((ids >= 0) & (slot < 0)).any(axis=1))[0]
    toks = np.union1d(rng.choice(w.N, size=12, replace=False), lost[:4])
    ref = oracle.token_dx(inp["x"][toks], inp["W_r"], lambda e: (inp["W_g"][e], inp["W_u"][e], inp["W_d"][e]),
                          dY[toks], ids[toks], wts[toks], slot[toks], norm=w.norm, reject_policy=w.reject_policy,
                          b_r=inp.get("b_r"), bf16=True)
    got = g["dx"].index_select(0, torch.from_numpy(toks).cuda()).cpu().numpy().astype(np.float64)
    err, row = parity.rel_err(got, ref), parity.row_rel_err(got, ref)
    worst["dx"] = row
    assert err <= 5e-3 and row <= 1e-2, (name, "dx", err, row)
    print(f"{name}: largest per-row error {worst}, experts {experts} with {acc_rows[experts].tolist()} rows, "
          f"{toks.size} tokens ({min(lost.size, 4)} with a rejected path)")
