"""Host-side accounting of bench.py, on CPU: the roofline numerators against
hand-computed closed forms, the launch counts against the kernel lists of the
committed launch summaries, the committed-traffic lookup and the clock-record
parsing."""
import json

import pytest

import bench
import seeded_inputs as si

W = si.WORKLOADS


def test_mixtral_gate_up_work():
    w = W["mixtral_bf16"]
    # 2 A d (2 d_f) with A = N k = 8192 routed rows, no shared expert
    assert bench.gate_up_flops(w, 8192) == 2 * 8192 * 4096 * 2 * 14336 == 1_924_145_348_608
    # weights of the 8 touched experts (bf16), gathered rows read and h written
    # (bf16), Y zeroed (fp32)
    want = 8 * 2 * 14336 * 4096 * 2 + 8192 * (4096 + 14336) * 2 + 4096 * 4096 * 4
    assert want == 2_248_146_944
    assert bench.gate_up_bytes(w, 8192, 8) == want


def test_shared_expert_terms():
    w = W["deepseek_shared_bf16"]
    A = 1000
    base = 2.0 * A * w.d * 2 * w.d_f
    assert bench.gate_up_flops(w, A) == base + 2.0 * w.N * w.d * 2 * w.d_f_shared
    # the step adds the router and three matrices per expert and shared expert
    assert bench.step_flops(w, A) == (2.0 * w.N * w.d * w.E + 2.0 * A * 3 * w.d * w.d_f
                                      + 2.0 * w.N * 3 * w.d * w.d_f_shared)
    b0 = bench.gate_up_bytes(w, A, 10)
    assert b0 == (10 * 2.0 * w.d_f * w.d * 2 + A * (w.d + w.d_f) * 2 + w.N * w.d * 4.0
                  + 2.0 * w.d_f_shared * w.d * 2 + w.N * (w.d + w.d_f_shared) * 2)


def test_ffma_peak():
    # 148 SMs x 128 FP32 lanes x 2 FLOP per FFMA at 1965 MHz
    assert bench.ffma_peak_tflops(1965.0) == pytest.approx(74.45, abs=0.01)


def test_forward_launch_counts_match_the_launch_lists():
    # profiles/launches_mixtral_bf16.md and launches_qwen3_skew_bf16.md: 8
    # kernels per forward pass (scores, top-k, hist, scan, assign, gather,
    # gate/up, down)
    assert bench.kernels_per_step(W["mixtral_bf16"], sharded=False) == 8
    assert bench.kernels_per_step(W["qwen3_skew_bf16"], sharded=False) == 8
    # acceptance by weight: placement, select + numbering and the per-token
    # pass replace the slot assignment (10 kernels per pass)
    wq = W["qwen3_skew_bf16"].scaled("qwen3_weight", accept_order=1)
    assert bench.kernels_per_step(wq, sharded=False) == 10
    # the sharded group adds the count kernel
    assert bench.kernels_per_step(W["mixtral_bf16"], sharded=True) == 9


def test_backward_launch_counts_match_the_backward_profile():
    # profiles/backward_all_configs.md: launches per call 30 / 31 / 50
    assert bench.backward_kernels(W["mixtral_bf16"]) == 30
    assert bench.backward_kernels(W["qwen3_skew_bf16"]) == 31
    assert bench.backward_kernels(W["deepseek_shared_bf16"]) == 50


def test_committed_traffic_follows_the_kernel_source(monkeypatch):
    with open(bench.TRAFFIC_FILE) as f:
        ent = json.load(f)["gate_up:mixtral_bf16"]
    if ent["source_sha256_16"] == bench.kernel_source_hash():
        assert bench.committed_traffic("gate_up", "mixtral_bf16") == ent["bytes_per_launch"]
    assert bench.committed_traffic("gate_up", "no_such_workload") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.committed_traffic("gate_up", "mixtral_bf16") is None


def test_committed_traffic_is_close_to_the_algorithmic_bytes():
    with open(bench.TRAFFIC_FILE) as f:
        ent = json.load(f)["gate_up:mixtral_bf16"]
    alg = bench.gate_up_bytes(W["mixtral_bf16"], 8192, 8)
    assert 1.0 <= ent["bytes_per_launch"] / alg < 1.05


def test_clock_record_parsing():
    s = bench.ClockSampler(0)
    s.proc = object()
    s.out = "\n".join([
        "0, 1965, 1965, 812.3, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 1001.2, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ])
    got = s.summary()
    assert got["sm_mhz"] == 1965.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"] and got["samples"] == 3
    s.out = "0, 1200, 1965, 700, 0x0000000000000020, Not Active, Active, Not Active, Not Active"
    assert bench.ClockSampler.summary(s)["reasons"] == ["hw_thermal_slowdown"]
    none = bench.ClockSampler(0)
    assert none.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_per_config_summary_keeps_the_contract_keys():
    line = {"value": 1.0, "unit": "tokens/s", "ms_per_step": 2.0, "steps": 20, "warmup": 5, "dtype": "bf16",
            "config": {"workload": "x"}, "stages_ms": {}, "gpu_launches": 8, "clocks": {}, "routing": {},
            "roofline": {"kernel": "k", "bound": "tensor", "achieved": 1.0, "peak": 2.0, "unit": "TFLOP/s",
                         "frac": 0.5, "traffic": None, "peak_source": "fallback", "avg_launch_ms": 1.0,
                         "hbm_frac": 0.1, "tensor_frac": 0.5, "extra": 1},
            "e2e": {"value": 1.0, "unit": "tokens/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 2,
                    "ms_per_step": 3.0, "how": "x"}, "other": 1}
    out = bench.per_config_summary(line)
    assert "other" not in out and "extra" not in out["roofline"] and "how" not in out["e2e"]
    assert out["roofline"]["frac"] == 0.5 and out["roofline"]["tensor_frac"] == 0.5
    assert set(out["e2e"]) == {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step", "ms_per_step"}

