"""The C-ABI library on a host without a GPU: it loads, exports every entry
point the header declares, and its host-side logic (capacity, workspace
layout, argument checks) behaves as documented.  No call here reaches a
CUDA device."""
import ctypes
import math

import pytest

import oracle
import sparse_mixture_experts_25_b200 as moe


def test_library_exports_every_declared_symbol():
    names = moe.declared_symbols()
    assert {"moe_capacity", "moe_workspace_size", "moe_route", "moe_dispatch", "moe_expert_ffn",
            "moe_combine", "moe_forward", "moe_get_stats", "moe_status_string"} <= set(names)
    lib = moe.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_struct_sizes_match_the_header_layout():
    assert ctypes.sizeof(moe.Params) == 64
    assert ctypes.sizeof(moe.Stats) == 13 * 8 + 2 * 8 + 2 * 4 + 8 + 8 + 8
    assert ctypes.sizeof(moe.WsLayout) == 19 * 8


@pytest.mark.parametrize("c,N,k,E", [
    (1.25, 1024, 1, 8), (1.25, 1000, 1, 8), (1.0, 4, 2, 3), (1.25, 8192, 8, 128),
    (1.1, 1000, 1, 11), (1.25, 1001, 1, 8), (0.0, 4096, 2, 8), (-1.0, 77, 2, 8),
    (2.0, 3, 1, 8), (0.3, 10, 1, 1000), (1.5, 4096, 8, 256), (0.9999999, 1000, 1, 10),
    (1.0000000001, 1000, 1, 10), (3.7, 12345, 6, 97),
])
def test_capacity_matches_oracle(c, N, k, E):
    p = moe.params(N, 64, 64, E, k, c=c)
    assert moe.moe_capacity(p) == oracle.capacity(c, N, k, E)


def test_capacity_printed_examples():
    assert moe.moe_capacity(moe.params(1024, 64, 64, 8, 1, c=1.25)) == 160
    assert moe.moe_capacity(moe.params(1000, 64, 64, 8, 1, c=1.25)) == 157
    assert moe.moe_capacity(moe.params(4, 64, 64, 3, 2, c=1.0)) == 3


def test_workspace_layout_regions():
    p = moe.params(4096, 4096, 14336, 8, 2, dtype=moe.MOE_BF16)
    L = moe.moe_workspace_layout(p)
    assert moe.moe_workspace_size(p) == L["total"]
    regions = sorted((v, k) for k, v in L.items() if k != "total")
    for (o, _), (o2, _) in zip(regions, regions[1:]):
        assert o % 256 == 0 and o2 >= o
    assert L["h"] - L["x_perm"] >= 4096 * 2 * 4096 * 2
    assert L["total"] - L["h"] >= 4096 * 2 * 14336 * 2
    ps = moe.params(64, 4096, 2048, 8, 2, dtype=moe.MOE_BF16, d_f_shared=2048)
    Ls = moe.moe_workspace_layout(ps)
    assert Ls["scratch"] - Ls["h_shared"] >= 64 * 2048 * 2


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(k=9), moe.MOE_ERR_INVALID_ARG),
    (dict(N=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(norm=7), moe.MOE_ERR_INVALID_ARG),
    (dict(dtype=5), moe.MOE_ERR_INVALID_ARG),
    (dict(norm=moe.MOE_NORM_WLR, theta=1.5), moe.MOE_ERR_INVALID_ARG),
    (dict(d=100), moe.MOE_ERR_UNSUPPORTED),
    (dict(d_f=36), moe.MOE_ERR_UNSUPPORTED),
    (dict(E_r=2000, k=2), moe.MOE_ERR_UNSUPPORTED),
    (dict(c=float("nan")), moe.MOE_ERR_INVALID_ARG),
    (dict(reject_policy=3), moe.MOE_ERR_INVALID_ARG),
    (dict(accept_order=2), moe.MOE_ERR_INVALID_ARG),
    # rerouting: 1 <= depth <= min(E_r - k, 32 - k); not with WLR or acceptance by weight
    (dict(reject_policy=2), moe.MOE_ERR_INVALID_ARG),
    (dict(reject_policy=2, reroute_depth=7), moe.MOE_ERR_INVALID_ARG),
    (dict(reject_policy=2, E_r=64, k=30, reroute_depth=3), moe.MOE_ERR_INVALID_ARG),
    (dict(reject_policy=2, reroute_depth=2, norm=moe.MOE_NORM_WLR, theta=0.3), moe.MOE_ERR_UNSUPPORTED),
    (dict(reject_policy=2, reroute_depth=2, accept_order=1), moe.MOE_ERR_UNSUPPORTED),
])
def test_invalid_params_are_rejected_on_the_host(kw, status):
    base = dict(N=16, d=64, d_f=64, E_r=8, k=2)
    base.update(kw)
    p = moe.params(**base)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_workspace_size(p)
    assert ei.value.status == status


def test_missing_workspace_is_reported_before_any_device_work():
    p = moe.params(16, 64, 64, 8, 2)
    r = moe.lib().moe_forward(ctypes.byref(p), None, None, None, None, None, None, None, None,
                              None, None, None, None, None)
    assert r == moe.MOE_ERR_WORKSPACE
    r = moe.lib().moe_dispatch(ctypes.byref(p), None, None, 0, None, None, None, None, None, None,
                               None, None)
    assert r == moe.MOE_ERR_WORKSPACE
    # router of more than 256 experts is not implemented by the fused router kernel
    p = moe.params(16, 64, 64, 512, 2)
    r = moe.lib().moe_route(ctypes.byref(p), None, None, None, None, None, None, None, None, None)
    assert r == moe.MOE_ERR_UNSUPPORTED


def test_wait_selftest_limits_are_checked_on_the_host():
    p = moe.params(16, 64, 64, 8, 2)
    for bad in (0, 999_999, 5_000_000_001):
        r = moe.lib().moe_selftest_wait_timeout(ctypes.byref(p), None, bad, None)
        assert r == moe.MOE_ERR_INVALID_ARG
    r = moe.lib().moe_selftest_wait_timeout(ctypes.byref(p), None, 50_000_000, None)
    assert r == moe.MOE_ERR_WORKSPACE


def test_reroute_workspace_regions_and_refusals():
    p = moe.params(1000, 64, 64, 16, 4, c=1.0, reject_policy=moe.MOE_REJECT_REROUTE, reroute_depth=5)
    L = moe.moe_workspace_layout(p)
    assert L["cand_w"] - L["cand"] >= 1000 * 5 * 4 and L["rr_e"] - L["cand_w"] >= 1000 * 5 * 4
    assert L["rr_slot"] - L["rr_e"] >= 1000 * 4 * 4 and L["scratch"] - L["rr_slot"] >= 1000 * 4 * 4
    p0 = moe.params(1000, 64, 64, 16, 4, c=1.0)
    L0 = moe.moe_workspace_layout(p0)
    assert L0["cand"] == L0["cand_w"] == L0["rr_e"] == L0["rr_slot"] == L0["scratch"]
    assert moe.moe_workspace_size(p) > moe.moe_workspace_size(p0)
    lib = moe.lib()
    fake = ctypes.c_void_p(256)
    assert lib.moe_forward_begin(ctypes.byref(p), fake, fake, None, None, None, fake, None) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_dispatch_noalloc(ctypes.byref(p), fake, fake, 1, fake, fake, fake, fake, None, None,
                                    None) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_backward_workspace_size(ctypes.byref(p), None, ctypes.byref(ctypes.c_size_t())) == \
        moe.MOE_ERR_UNSUPPORTED


def test_acceptance_by_weight_is_refused_where_it_is_not_built():
    # one routing group over ranks would need every rank's weights, and the
    # no-allocation dispatch has no room for the ranking arrays
    p = moe.params(16, 64, 64, 8, 2, c=1.0, accept_order=moe.MOE_ACCEPT_WEIGHT)
    L = moe.lib()
    assert L.moe_forward_begin(ctypes.byref(p), None, None, None, None, None, None, None) == \
        moe.MOE_ERR_UNSUPPORTED
    assert L.moe_dispatch_noalloc(ctypes.byref(p), None, None, 1, None, 16, None, None, None, None,
                                  None) == moe.MOE_ERR_UNSUPPORTED


def test_soft_moe_params_are_checked_on_the_host():
    assert ctypes.sizeof(moe.SoftParams) == 32
    L = moe.lib()
    n = ctypes.c_size_t(0)
    for kw, status in ((dict(dtype=moe.MOE_F32), moe.MOE_ERR_UNSUPPORTED),   # bf16 contractions only
                       (dict(N=100), moe.MOE_ERR_UNSUPPORTED),                # 16-byte operand rows
                       (dict(E_r=3, p=3), moe.MOE_ERR_UNSUPPORTED),           # S = 9 slots
                       (dict(p=0), moe.MOE_ERR_INVALID_ARG),
                       (dict(d=0), moe.MOE_ERR_INVALID_ARG)):
        args = dict(N=64, d=64, d_f=32, E_r=8, p=2)
        args.update(kw)
        sp = moe.soft_params(**args)
        assert L.moe_soft_workspace_size(ctypes.byref(sp), ctypes.byref(n)) == status, kw
    sp = moe.soft_params(64, 64, 32, 8, 2)
    assert L.moe_soft_workspace_size(ctypes.byref(sp), ctypes.byref(n)) == moe.MOE_OK and n.value > 0
    assert L.moe_soft_forward(ctypes.byref(sp), None, None, None, None, None, None, None, None) == \
        moe.MOE_ERR_WORKSPACE


def test_ranked_dispatch_and_row_gather_check_arguments_on_the_host():
    L = moe.lib()
    p = moe.params(16, 64, 64, 8, 2, c=1.0)
    # rank out of range, missing counts, C < 1, a group smaller than the shard
    for rank, n_ranks, counts, N_group, C in ((2, 2, 16, 32, 4), (0, 2, None, 32, 4), (0, 2, 16, 32, 0),
                                              (0, 2, 16, 8, 4)):
        r = L.moe_dispatch_ranked(ctypes.byref(p), counts, rank, n_ranks, N_group, C, 16, 256, None)
        assert r == moe.MOE_ERR_INVALID_ARG, (rank, n_ranks, counts, N_group, C)
    assert L.moe_dispatch_ranked(ctypes.byref(p), 16, 0, 2, 32, 4, 16, None, None) == moe.MOE_ERR_WORKSPACE
    pw = moe.params(16, 64, 64, 8, 2, c=1.0, accept_order=moe.MOE_ACCEPT_WEIGHT)
    assert L.moe_dispatch_ranked(ctypes.byref(pw), 16, 0, 2, 32, 4, 16, 256, None) == moe.MOE_ERR_UNSUPPORTED
    # row sizes must be whole 16-byte words; nothing to do for zero rows
    assert L.moe_gather_rows(16, 16, 4, 24, 16, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_gather_rows(16, 16, -1, 32, 16, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_gather_rows(None, None, 0, 32, None, None) == moe.MOE_OK


def test_status_strings():
    for s in range(7):
        assert moe.moe_status_string(s)
    assert "non-finite" in moe.moe_status_string(moe.MOE_ERR_NONFINITE)


def test_host_tensors_are_refused_by_the_binding():
    torch = pytest.importorskip("torch")
    p = moe.params(4, 64, 64, 8, 2)
    with pytest.raises(ValueError):
        moe.moe_forward(p, torch.zeros(4, 64), None, None, None, None, None, None, None, None, None,
                        None, None, stream=0)


def test_backward_checks_arguments_on_the_host():
    L = moe.lib()
    assert ctypes.sizeof(moe.Grads) == 9 * 8
    p = moe.params(16, 64, 64, 8, 2, c=1.0)
    sz = ctypes.c_size_t()
    # fp32 layers keep fp32 rows only (no transposed operands); E_r above the
    # router kernel's limit has no backward
    p32 = moe.params(16, 64, 64, 8, 2, c=1.0, dtype=moe.MOE_F32)
    assert 0 < moe.moe_backward_workspace_size(p32) < moe.moe_backward_workspace_size(p)
    assert L.moe_backward_workspace_size(ctypes.byref(moe.params(16, 64, 64, 300, 2)), None,
                                         ctypes.byref(sz)) == moe.MOE_ERR_UNSUPPORTED
    good = [0, 4, 4, 8, 12, 16, 20, 24, 28]
    n_any = moe.moe_backward_workspace_size(p)
    n = moe.moe_backward_workspace_size(p, good)
    assert n >= 8 * 64 * 64 * 2 * 3            # the transposed expert weights alone
    # C = 4 rows per expert at most: one 64-wide K block either way
    assert n == n_any
    # the bound grows with the capacity; a routing with a long expert needs more
    big = moe.params(256, 64, 64, 8, 2)
    skew = [0, 200, 200, 200, 200, 200, 200, 200, 200]
    even = [0, 25, 50, 75, 100, 125, 150, 175, 200]
    assert moe.moe_backward_workspace_size(big, skew) > moe.moe_backward_workspace_size(big, even)
    assert moe.moe_backward_workspace_size(big) >= moe.moe_backward_workspace_size(big, skew)
    arr_bad = (ctypes.c_int32 * 9)(*([0, 5, 3] + good[3:]))
    assert L.moe_backward_workspace_size(ctypes.byref(p), arr_bad, ctypes.byref(sz)) == moe.MOE_ERR_INVALID_ARG
    fake = 4096                                  # aligned, never dereferenced: the checks come first
    g = moe.Grads(*([fake] * 9))

    def call(offsets, ws=fake, bws=fake, grads=g, aux=0.0, nbytes=n):
        arr = (ctypes.c_int32 * len(offsets))(*offsets)
        return L.moe_backward(ctypes.byref(p), aux, arr, fake, fake, None, fake, fake, fake, None, None, None,
                              fake, ws, ctypes.byref(grads) if grads is not None else None, bws, nbytes, None)

    assert call(good, ws=None) == moe.MOE_ERR_WORKSPACE
    assert call(good, bws=fake + 8) == moe.MOE_ERR_WORKSPACE
    assert call(good, nbytes=n - 1) == moe.MOE_ERR_WORKSPACE
    assert call(good, grads=None) == moe.MOE_ERR_INVALID_ARG
    assert call(good, aux=float("nan")) == moe.MOE_ERR_INVALID_ARG
    assert call([1] + good[1:]) == moe.MOE_ERR_INVALID_ARG             # does not start at 0
    assert call([0, 4, 3] + good[3:]) == moe.MOE_ERR_INVALID_ARG       # decreasing
    assert call(good[:-1] + [33]) == moe.MOE_ERR_INVALID_ARG           # more rows than N k
    missing = moe.Grads(*([fake] * 3 + [None] + [fake] * 5))          # dW_g missing
    assert call(good, grads=missing) == moe.MOE_ERR_INVALID_ARG
    ps = moe.params(16, 64, 64, 8, 2, d_f_shared=64)
    arr = (ctypes.c_int32 * 9)(*good)
    no_shared = moe.Grads(*([fake] * 6 + [None] * 3))
    assert L.moe_backward(ctypes.byref(ps), 0.0, arr, fake, fake, None, fake, fake, fake, fake, fake, fake, fake,
                          fake, ctypes.byref(no_shared), fake, 1 << 40, None) == moe.MOE_ERR_INVALID_ARG


def test_backward_of_an_empty_batch_needs_no_dx():
    # an empty dx tensor has no storage (a null pointer): N = 0 must pass the
    # argument checks without it (on a host without a GPU the call then fails
    # in CUDA; with a GPU it would write to the fake addresses, so it is skipped)
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("fake device addresses are only safe without a GPU")
    L = moe.lib()
    p = moe.params(0, 64, 64, 8, 2)
    fake = 4096
    g = moe.Grads(None, *([fake] * 8))
    arr = (ctypes.c_int32 * 9)(*([0] * 9))
    r = L.moe_backward(ctypes.byref(p), 0.0, arr, None, None, None, None, None, None, None, None, None, None,
                       fake, ctypes.byref(g), fake, 0, None)
    assert r not in (moe.MOE_ERR_INVALID_ARG, moe.MOE_ERR_WORKSPACE)


def test_backward_binding_checks_the_offsets_shape():
    p = moe.params(16, 64, 64, 8, 2)
    with pytest.raises(ValueError):
        moe.moe_backward_workspace_size(p, [0, 1, 2])
    with pytest.raises(ValueError):
        moe.moe_backward(p, [0] * 8, None, None, None, None, None, None, None, None, None, None, None, {}, None)
