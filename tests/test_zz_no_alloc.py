"""moe_dispatch_noalloc, the dispatch entry point that allocates nothing.

It exists for callers that cannot allocate device memory where they dispatch
(a memory pool that may not grow, an allocator not reachable from the call
site, or a call site that must not risk the device synchronisation cudaMalloc
can cause).  Its scratch lives in a fixed buffer inside the library, shared
by every call.  This file is collected last so that a run that stops at the
first failure has already run every other test; it also passes on its own in
a fresh process.
"""
import numpy as np
import pytest

import seeded_inputs as si
from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_25_b200 as moe  # noqa: E402


def _routed(w):
    inp = si.inputs(w)
    dev = {k: parity.to_dev(v) for k, v in inp.items()}
    p = parity.params_of(w)
    ws = torch.zeros(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    ids = torch.empty(w.N, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(w.N, w.k, dtype=torch.float32, device="cuda")
    moe.moe_route(p, dev["x"], dev["W_r"], dev.get("b_r"), dev.get("lat"), ids, wt, None, ws)
    return p, dev, ids, wt, ws


def _outputs(w, dtype):
    Nk = w.N * w.k
    return dict(slot=torch.full((w.N, w.k), -7, dtype=torch.int32, device="cuda"),
                offsets=torch.full((w.E + 1,), -7, dtype=torch.int32, device="cuda"),
                st=torch.full((Nk,), -7, dtype=torch.int32, device="cuda"),
                sw=torch.full((Nk,), -7.0, dtype=torch.float32, device="cuda"),
                x_perm=torch.zeros(Nk, w.d, dtype=dtype, device="cuda"))


def _compare(a, b, total):
    for key in ("slot", "offsets"):
        assert torch.equal(a[key], b[key]), key
    for key in ("st", "sw", "x_perm"):
        assert torch.equal(a[key][:total], b[key][:total]), key


def test_noalloc_dispatch_matches_workspace_dispatch_on_two_calls_in_a_row():
    # two different batches back to back: the second call must not depend on
    # what the first left in the shared scratch buffer
    cases = [si.WORKLOADS["qwen3_skew_bf16"].scaled("noalloc_a", N=1024, d=256, d_f=192, E=32, k=4),
             si.WORKLOADS["switch_top1_f32"].scaled("noalloc_b", N=777, d=64, d_f=64, E=8, k=1, c=0.5)]
    for w in cases:
        p, dev, ids, wt, ws = _routed(w)
        C = moe.moe_capacity(p)
        ref = _outputs(w, dev["x"].dtype)
        moe.moe_dispatch(p, ids, wt, C, ref["slot"], ref["offsets"], ref["st"], ref["sw"], dev["x"],
                         ref["x_perm"], ws)
        for _ in range(2):
            out = _outputs(w, dev["x"].dtype)
            moe.moe_dispatch_noalloc(p, ids, wt, C, out["slot"], out["offsets"], out["st"], out["sw"],
                                     dev["x"], out["x_perm"])
            torch.cuda.synchronize()
            total = int(ref["offsets"][-1])
            _compare(out, ref, total)
        # the capped case really rejected paths, so slots of -1 were exercised
        if w.c > 0:
            assert (ref["slot"] < 0).any()


def test_noalloc_dispatch_leaves_free_device_memory_unchanged():
    """After a first call (which may load the library and reserve its static
    array), further calls change nothing in the device's free memory."""
    w = si.WORKLOADS["qwen3_skew_bf16"].scaled("noalloc_mem", N=2048, d=128, d_f=64, E=64, k=8)
    p, dev, ids, wt, ws = _routed(w)
    C = moe.moe_capacity(p)
    out = _outputs(w, dev["x"].dtype)
    args = (p, ids, wt, C, out["slot"], out["offsets"], out["st"], out["sw"], dev["x"], out["x_perm"])
    moe.moe_dispatch_noalloc(*args)           # warm-up: the one-time set-up happens here at the latest
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        moe.moe_dispatch_noalloc(*args)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_dispatch_rejects_sizes_beyond_its_buffer():
    p = moe.params(1 << 20, 64, 64, 1024, 1)
    dummy = torch.zeros(8, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_dispatch_noalloc(p, dummy, dummy, 1, dummy, dummy, dummy, dummy, None, None)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    assert "static buffer" in str(ei.value)
