"""Failure detection on the GPU without faulting it.

The library's device waits (mbarrier waits of the tensor-core GEMMs) are
bounded: on expiry they record a timeout in the workspace counters and the
CTA returns, so the host sees MOE_ERR_TIMEOUT and the CUDA context stays
usable.  Here the wait is made to run out on purpose through the self-test
entry point (a barrier nothing arrives on, 50 ms limit); then the same
context runs the layer and is checked against the oracle.
"""
import time

import pytest

import seeded_inputs as si
from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - GPU tests need a device
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_25_b200 as moe  # noqa: E402


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    w = si.WORKLOADS["mixtral_bf16"].scaled("after_timeout", N=256, d=128, d_f=256)
    p = parity.params_of(w)
    ws = torch.zeros(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moe.moe_selftest_wait_timeout(p, ws, 50_000_000)
    status, stats = moe.moe_get_stats(p, ws)
    dt = time.perf_counter() - t0
    assert status == moe.MOE_ERR_TIMEOUT
    assert stats["device_error"] & 1
    assert 0.04 < dt < 5.0, dt
    # the context is intact: the layer runs and matches the oracle
    inp = si.inputs(w)
    out = parity.gpu_forward(w, inp)
    assert out["status"] == moe.MOE_OK
    parity.check_dispatch(w, out["rec"], out["stats"])
    parity.check_rows(w, inp, out["rec"], out["Y"])
