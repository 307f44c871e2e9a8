"""Expert parallelism on one GPU: R ranks' steps run in one process with the
collectives replaced by copies (expert_parallel.emulate), and one rank through
a one-rank NCCL group (ExpertParallelLayer.forward).  The routing records and
outputs equal the single-GPU layer on the whole batch."""
import os
import socket

import numpy as np
import pytest

import seeded_inputs as si
from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - GPU tests need a device
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_25_b200 as moe  # noqa: E402
from sparse_mixture_experts_25_b200 import expert_parallel as ep  # noqa: E402
from sparse_mixture_experts_25_b200 import sharded  # noqa: E402
from tests import ep_host_plan  # noqa: E402

W = si.WORKLOADS
CASES = {
    "qwen3_skewed_capped": W["qwen3_skew_bf16"].scaled("ep_qwen3", N=1024, d=256, d_f=192, E=32, k=4),
    "deepseek_shared": W["deepseek_shared_bf16"].scaled("ep_deepseek", N=384, d=448, d_f=128, E=64, k=6,
                                                        d_f_shared=192),
    "mixtral_pairs": W["mixtral_bf16"].scaled("ep_mixtral", N=1600, d=320, d_f=384, E=8, k=2),
    "switch_f32_capped": W["switch_top1_f32"].scaled("ep_switch", N=1000, d=72, d_f=96),
}


def _ranks(w, R, dev):
    layers, xs = [], []
    El = w.E // R
    for r in range(R):
        lo, hi = sharded.shard_range(w.N, r, R)
        p = parity.params_of(w.scaled(w.name, N=hi - lo))
        sl = slice(r * El, (r + 1) * El)
        shared = (dev["Ws_g"], dev["Ws_u"], dev["Ws_d"]) if w.d_f_shared else None
        layers.append(ep.ExpertParallelLayer(p, r, R, w.N, dev["W_r"], dev["W_g"][sl], dev["W_u"][sl],
                                             dev["W_d"][sl], b_r=dev.get("b_r"), lat=dev.get("lat"),
                                             shared=shared))
        xs.append(dev["x"][lo:hi].contiguous())
    return layers, xs


@pytest.mark.parametrize("path", ["collectives", "fused"])
@pytest.mark.parametrize("name,R", [("qwen3_skewed_capped", 2), ("qwen3_skewed_capped", 4),
                                    ("deepseek_shared", 4), ("mixtral_pairs", 2), ("switch_f32_capped", 4)])
def test_expert_parallel_emulated(name, R, path):
    """R ranks in one process: with the rows moved by (emulated) all-to-all
    collectives, or written straight into the owners' expert-major buffers and
    read back from them (the fused exchange, the owners' buffers local here)."""
    w = CASES[name]
    inp = si.inputs(w)
    full = parity.gpu_forward(w, inp)
    dev = full["dev"]
    layers, xs = _ranks(w, R, dev)
    Ys = [torch.full((x.shape[0], w.d), float("nan"), device="cuda") for x in xs]
    (ep.emulate if path == "collectives" else ep.emulate_peer)(layers, xs, Ys)
    torch.cuda.synchronize()
    # the device plan against the host restatement
    counts_all = np.stack([L.counts.cpu().numpy() for L in layers])
    acc = ep_host_plan.accepted_counts(counts_all, layers[0].C)
    rows = ep_host_plan.send_rows(acc, R)
    for r, L in enumerate(layers):
        send, recv = L.split_sizes()
        assert send == [int(v) for v in rows[r]] and recv == [int(v) for v in rows[:, r]]
        index, offsets = ep_host_plan.regroup(acc, r, R)
        np.testing.assert_array_equal(L.local_offsets.cpu().numpy(), offsets)
        if path == "collectives":
            np.testing.assert_array_equal(L.regroup[:index.size].cpu().numpy(), index)
        views = moe.workspace_views(L.p, L.ws)
        np.testing.assert_array_equal(views["acc"].cpu().numpy(), acc[r])
    ids = np.concatenate([moe.workspace_views(L.p, L.ws)["ids"].cpu().numpy() for L in layers])
    np.testing.assert_array_equal(ids, full["rec"]["ids"])
    slot = np.concatenate([moe.workspace_views(L.p, L.ws)["slot"].cpu().numpy() for L in layers])
    np.testing.assert_array_equal(slot, full["rec"]["slot"])
    if full["stats"]["rejected"]:
        assert (slot < 0).any()
    # the owners run the unfused expert kernels: outputs against the oracle on
    # the (identical) routing records, at the layer's tolerance
    Y = np.concatenate([y.cpu().numpy() for y in Ys]).astype(np.float64)
    parity.check_rows(w, inp, full["rec"], Y)


def test_expert_parallel_forward_one_rank_nccl():
    """ExpertParallelLayer.forward through torch.distributed (NCCL, one rank)."""
    import torch.distributed as dist
    w = CASES["qwen3_skewed_capped"]
    inp = si.inputs(w)
    full = parity.gpu_forward(w, inp)
    dev = full["dev"]
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        (layer,), (x,) = _ranks(w, 1, dev)
        Y = torch.full((w.N, w.d), float("nan"), device="cuda")
        layer.forward(x, Y)
        torch.cuda.synchronize()
        parity.check_rows(w, inp, full["rec"], Y.cpu().numpy().astype(np.float64))
    finally:
        dist.destroy_process_group()
