"""Benchmark of the sparse-MoE layer forward pass on B200.

Default workload: the Mixtral-shaped bf16 layer (T = 4096 tokens, d = 4096,
d_f = 14336, E_r = 8, k = 2, renormalised top-2, no capacity limit), seeded
synthetic inputs.  One step = one moe_forward (router, softmax, top-k,
dispatch, gate/up GEMM + SwiGLU, down GEMM + combine) over the batch.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  --impl reference times the CPU oracle on the
host cores on a bounded sample of the same workload.  Under torchrun each
rank runs its own token batch (weak scaling; the uncapped layer needs no
exchange between ranks), timed on the device, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import seeded_inputs as si  # noqa: E402

METRIC = "MoE-layer fwd tokens/s; achieved TFLOP/s or HBM GB/s as fraction of B200 peak"
WORKLOAD = "mixtral_bf16"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def kernels_per_step(w: si.Workload, sharded: bool) -> int:
    """libmoe kernels one forward launches for this workload."""
    if w.dtype == si.DT_BF16 and w.E % 4 == 0:
        router = 2                      # score GEMM (tensor cores) + warp top-k
    else:
        router = 1                      # fused FFMA router
    dispatch = 5 if sharded else 4      # hist, scan(s), assign, gather
    if w.accept_order == 1:
        dispatch += 2                   # placement, select + numbering, per-token pass replace assign
    if w.reject_policy == 2:
        dispatch += 3 * w.reroute_depth + 2   # offer, scan, assign per round; final offsets; rows
    experts = 2 if w.dtype == si.DT_BF16 else 3   # fp32 layers zero Y in the router or a kernel
    if w.dtype != si.DT_BF16 and not sharded:
        experts = 2
    return router + dispatch + experts


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# algorithmic work of one step (the roofline numerators)
# ---------------------------------------------------------------------------
def gate_up_flops(w: si.Workload, accepted: int) -> float:
    """2 * A * d * (2 d_f) for the routed rows, plus the shared expert's N rows."""
    f = 2.0 * accepted * w.d * 2 * w.d_f
    if w.d_f_shared:
        f += 2.0 * w.N * w.d * 2 * w.d_f_shared
    return f


def step_flops(w: si.Workload, accepted: int) -> float:
    """Router 2 N d E_r + experts 2 A 3 d d_f + shared 2 N 3 d d_sh (p2 ch. 36.5 cost model)."""
    f = 2.0 * w.N * w.d * w.E + 2.0 * accepted * 3 * w.d * w.d_f
    if w.d_f_shared:
        f += 2.0 * w.N * 3 * w.d * w.d_f_shared
    return f


def gate_up_bytes(w: si.Workload, accepted: int, experts_touched: int) -> float:
    """Algorithmic HBM bytes of the gate/up launch: W_g and W_u of every
    expert with an accepted row, the gathered rows (A d) read and h (A d_f)
    written, Y zeroed (N d fp32); the shared expert adds its two matrices, x
    and h_shared."""
    s = 2 if w.dtype == si.DT_BF16 else 4
    b = experts_touched * 2.0 * w.d_f * w.d * s + accepted * (w.d + w.d_f) * s + w.N * w.d * 4.0
    if w.d_f_shared:
        b += 2.0 * w.d_f_shared * w.d * s + w.N * (w.d + w.d_f_shared) * s
    return b


# fp32 CUDA-core peak: 148 SMs x 128 FP32 lanes x 2 FLOP (FFMA) x the maximum SM clock
def ffma_peak_tflops(sm_mhz: float) -> float:
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK), "fallback"


def kernel_source_hash() -> str:
    p = os.path.join(ROOT, "sparse_mixture_experts_25_b200", "csrc", "gemm_tc.cu")
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, or None when there is none for that workload or the kernel source
    changed since the counters were taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        ent = t.get(f"{kernel}:{workload}")
        if ent and ent.get("source_sha256_16") == kernel_source_hash():
            return ent.get("bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.out = out
        return False

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle leg (the reference arm and the cpu_baseline key)
# ---------------------------------------------------------------------------
def oracle_sample(w: si.Workload, inp: dict, sample_tokens: int = 32):
    """Times the oracle on a bounded sample: routing and dispatch of the whole
    batch, and the expert outputs of `sample_tokens` tokens; returns the
    extrapolated whole-batch tokens/s and a description."""
    import oracle
    t0 = time.perf_counter()
    r = oracle.route(inp["x"], inp["W_r"], k=w.k, norm=w.norm, theta=w.theta, b_r=inp.get("b_r"),
                     lat=inp.get("lat"))
    C = oracle.capacity(w.c, w.N, w.k, w.E)
    if w.accept_order == 1:
        d = oracle.dispatch_priority(r["ids"], r["w"], E=w.E, C=C)
    else:
        d = oracle.dispatch(r["ids"], E=w.E, C=C)
    wc = oracle.reject_weights(r["ids"], r["w"], d["slot"], w.reject_policy)
    t1 = time.perf_counter()
    toks = np.linspace(0, w.N - 1, sample_tokens).astype(np.int64)
    Ws = (inp.get("Ws_g"), inp.get("Ws_u"), inp.get("Ws_d")) if w.d_f_shared else None
    oracle.forward_rows(inp["x"], r["ids"], wc, d["slot"], toks, inp["W_g"], inp["W_u"], inp["W_d"], Ws=Ws)
    t2 = time.perf_counter()
    per_batch = (t1 - t0) + (t2 - t1) * w.N / sample_tokens
    cores = si.host_threads()
    return {"value": w.N / per_batch, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"routing+dispatch of all {w.N} tokens ({t1 - t0:.2f} s) and expert outputs "
                       f"of {sample_tokens} tokens ({t2 - t1:.2f} s), extrapolated to {w.N} tokens"),
            "seconds": t2 - t0}


def run_reference(args):
    """The CPU oracle on the host cores: each step is one bounded sample of the
    workload (routing and dispatch of the whole batch, expert outputs of
    --ref-sample tokens).  steps / warmup / ms_per_step describe those samples
    as run; value is the whole-batch tokens/s extrapolated from them."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = si.WORKLOADS[args.workload]
    inp = si.inputs(w)
    steps = []
    for i in range(args.warmup + args.steps):
        s = oracle_sample(w, inp, sample_tokens=args.ref_sample)
        if i >= args.warmup:
            steps.append(s)
    val = statistics.median([s["value"] for s in steps])
    sample_ms = statistics.median([1000.0 * s["seconds"] for s in steps])
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sample_ms,
        "step": (f"one bounded sample of the workload: routing and dispatch of all {w.N} tokens and the expert "
                 f"outputs of {args.ref_sample} tokens"),
        "extrapolated": True,
        "extrapolated_ms_per_full_batch": 1000.0 * w.N / val,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args),
        "cpu_baseline": {k: steps[-1][k] for k in ("kind", "cores", "sample")} | {"value": val, "unit": "tokens/s"},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126 * 2**20


def input_bytes(w: si.Workload) -> int:
    """Bytes of the layer's inputs read every step: expert and router weights and x."""
    s = 2 if w.dtype == si.DT_BF16 else 4
    b = w.E * 3 * w.d * w.d_f * s + w.E * w.d * s + w.N * w.d * s
    if w.d_f_shared:
        b += 3 * w.d * w.d_f_shared * s
    return b


def flushes_l2(w: si.Workload) -> bool:
    return input_bytes(w) < 2 * L2_BYTES


def config_of(w: si.Workload, args):
    return {"workload": f"{w.name}: T={w.N} d={w.d} d_f={w.d_f} E_r={w.E} k={w.k}",
            "T": w.N, "d": w.d, "d_f": w.d_f, "E_r": w.E, "k": w.k,
            "norm": ["renorm", "fullprob", "wlr"][w.norm], "capacity_factor": w.c or None,
            "d_f_shared": w.d_f_shared, "seed": w.seed,
            "overflow": {"reject": ["zero", "renormalise", f"reroute (depth {w.reroute_depth})"][w.reject_policy],
                         "accept": ["token order", "largest weight"][w.accept_order]},
            "parallelism": (f"dp{args.gpus}: one routing group of {w.N} x {args.gpus} tokens, "
                            "per-expert request counts all-gathered once per step"
                            if args.gpus > 1 else "dp1"),
            "cuda_graph": bool(getattr(args, "graph", False)),
            "l2": (f"L2 flushed between timed steps (256 MiB write outside the per-step events); "
                   f"inputs {input_bytes(w) / 2**20:.1f} MiB" if flushes_l2(w) else
                   f"inputs larger than L2 ({input_bytes(w) / 1e9:.2f} GB of weights and x read every step)")}


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------
def run_gpu_soft(args):
    """Soft MoE layer (one GPU): one step = moe_soft_forward over the batch."""
    import torch
    ws_n, rank, local = dist_env()
    if ws_n > 1:
        raise SystemExit("the Soft MoE layer mixes every token into every slot: one GPU only")
    w = si.WORKLOADS[args.workload]
    names = ("x", "Phi", "W_g", "W_u", "W_d")
    inp = {n: si.tensor(w, n) for n in names}
    torch.cuda.set_device(local)
    import sparse_mixture_experts_25_b200 as moe
    d = {n: torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).cuda().view(torch.bfloat16)
         for n, v in inp.items()}
    sp = moe.soft_params(w.N, w.d, w.d_f, w.E, w.soft_p)
    wsb = torch.empty(moe.moe_soft_workspace_size(sp), dtype=torch.uint8, device="cuda")
    Y = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(x_dev, y_dev, ws_dev=wsb, st=stream):
        moe.moe_soft_forward(sp, x_dev, d["Phi"], d["W_g"], d["W_u"], d["W_d"], y_dev, ws_dev, st)

    for _ in range(args.warmup):
        step(d["x"], Y)
    if moe.moe_soft_check(sp, wsb) != moe.MOE_OK:
        raise RuntimeError("moe_soft_forward: a device wait gave up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        start.record(stream)
        for _ in range(args.steps):
            step(d["x"], Y)
        end.record(stream)
        torch.cuda.synchronize()
        time.sleep(0.2)
    ms_step = start.elapsed_time(end) / args.steps
    # end to end with host buffers
    from sparse_mixture_experts_25_b200.pipeline import HostPipeline
    x_host = torch.from_numpy(np.ascontiguousarray(inp["x"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty(w.N, w.d, dtype=torch.float32).pin_memory()
    pipe = HostPipeline(None, d, forward=lambda xd, yd, wsd, st: step(xd, yd, wsd, st),
                        ws_bytes=moe.moe_soft_workspace_size(sp), shape=(w.N, w.d))
    for _ in range(3):
        pipe.submit(x_host, y_host)
    pipe.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.h2d)
    for _ in range(args.steps):
        pipe.submit(x_host, y_host)
    pipe.compute.wait_stream(pipe.d2h)
    pipe.d2h.wait_stream(pipe.compute)
    e1.record(pipe.d2h)
    pipe.synchronize()
    e_ms = e0.elapsed_time(e1) / args.steps
    S = w.E * w.soft_p
    flops = 2.0 * w.N * S * w.d * 3 + 2.0 * S * 3 * w.d * w.d_f   # scores, D^T X, C Ys; experts
    peaks, peak_src = load_peaks()
    peak_tf = peaks["bf16_tflops"] if ms_step * args.steps < 1000 else peaks.get("bf16_tflops_sustained",
                                                                                   peaks["bf16_tflops"])
    achieved = flops / (ms_step * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": w.N / (ms_step * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64/Box-Muller; x~N(0,1), W~N(0,1/fan_in)); no dataset or checkpoint",
        "config": {"workload": f"{w.name}: Soft MoE T={w.N} d={w.d} d_f={w.d_f} E_r={w.E} slots={S}",
                   "T": w.N, "d": w.d, "d_f": w.d_f, "E_r": w.E, "slots_per_expert": w.soft_p,
                   "seed": w.seed, "parallelism": "dp1",
                   "l2": f"inputs larger than L2 ({input_bytes(w) / 1e9:.2f} GB of weights and x read every step)"},
        "roofline": {"kernel": "whole Soft MoE step (three slot contractions + slot experts)", "bound": "tensor",
                     "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved / peak_tf,
                     "traffic": None, "peak_source": f"{peak_src} bf16", "flops_per_step": flops},
        "e2e": {"value": w.N / (e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size()), "ms_per_step": e_ms},
        "gpu_launches": 14 * args.steps,   # scores, 2 column-statistics, dispatch weights, combine weights, x transpose, slot inputs, bf16, offsets, prefix, gate/up, down, transpose, combine
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


PER_CONFIG = ("switch_top1_f32", "qwen3_skew_bf16", "deepseek_shared_bf16", "wdmoe_decode_bf16")
EXPERT_TENSORS = ("W_g", "W_u", "W_d")


def device_inputs(w: si.Workload, rank: int, ws_n: int):
    """Host inputs of the layer's small tensors (x, router, bias, latencies,
    shared expert) and the same seeded expert weights generated one expert at
    a time straight into device tensors (a 22.6 GB layer never sits in host
    memory whole).  Returns (host dict of the small tensors, device dict)."""
    import torch

    small = ("x", "W_r", "b_r", "lat", "Ws_g", "Ws_u", "Ws_d")
    inp = si.inputs(w, names=small)
    if ws_n > 1:
        # rank r holds rows [r N, (r+1) N) of one routing group of N * ranks tokens
        inp["x"] = si.fill(w.seed, si.TID["x"], w.N * w.d, start=rank * w.N * w.d,
                           dtype=w.dt).reshape(w.N, w.d)

    def dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    d = {k: dev(v) for k, v in inp.items()}
    tdt = torch.bfloat16 if w.dtype == si.DT_BF16 else torch.float32
    for n in EXPERT_TENSORS:
        t = torch.empty(si.shape(w, n), dtype=tdt, device="cuda")
        for e in range(w.E):
            t[e].copy_(dev(si.tensor(w, n, expert=e)))
        d[n] = t
    return inp, d


def measure_forward(w: si.Workload, args, steps: int, warmup: int, cpu_base=None):
    """Device-timed moe_forward steps (inputs resident in HBM), stage times,
    the gate/up roofline and the end-to-end host-buffer leg for one workload;
    returns the JSON line (without printing)."""
    import torch
    import torch.distributed as dist
    import sparse_mixture_experts_25_b200 as moe

    ws_n, rank, local = dist_env()
    inp, d = device_inputs(w, rank, ws_n)
    p = moe.params(w.N, w.d, w.d_f, w.E, w.k, c=w.c, norm=w.norm, theta=w.theta, dtype=w.dtype,
                   d_f_shared=w.d_f_shared, reject_policy=w.reject_policy, accept_order=w.accept_order,
                   reroute_depth=w.reroute_depth)
    wsb = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    Y = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    sharded_group = ws_n > 1
    if sharded_group:
        from sparse_mixture_experts_25_b200 import sharded
        N_group = w.N * ws_n
        C_group = moe.moe_capacity(moe.params(N_group, w.d, w.d_f, w.E, w.k, c=w.c, norm=w.norm,
                                              theta=w.theta, dtype=w.dtype, d_f_shared=w.d_f_shared))
        counts = torch.empty(w.E, dtype=torch.int32, device="cuda")

    def step(x_dev, y_dev):
        if sharded_group:
            # one routing group over all ranks: exchange per-expert request counts
            sharded.forward_sharded(p, N_group, C_group, x_dev, d["W_r"], d["b_r"], d["lat"], d["W_g"],
                                    d["W_u"], d["W_d"], d["Ws_g"], d["Ws_u"], d["Ws_d"], y_dev, wsb,
                                    counts=counts, stream=stream)
        else:
            moe.moe_forward(p, x_dev, d["W_r"], d["b_r"], d["lat"], d["W_g"], d["W_u"], d["W_d"],
                            d["Ws_g"], d["Ws_u"], d["Ws_d"], y_dev, wsb, stream)

    for _ in range(warmup):
        step(d["x"], Y)
    torch.cuda.synchronize()
    status, stats = moe.moe_get_stats(p, wsb)
    if status != moe.MOE_OK:
        raise RuntimeError(f"moe_forward status: {moe.moe_status_string(status)}")
    accepted = int(stats["accepted"])

    # device-timed steps, inputs resident in HBM; stage events around each kernel group
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws_n > 1:
        dist.barrier()
    torch.cuda.synchronize()
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.int32, device="cuda") if flushes_l2(w) else None
    graph = None
    if args.graph and sharded_group:
        raise SystemExit("--graph times one GPU's step; the sharded group exchanges counts between ranks")
    if args.graph:
        # one step captured into a CUDA graph and replayed (fewer launch gaps)
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            moe.moe_forward(p, d["x"], d["W_r"], d["b_r"], d["lat"], d["W_g"], d["W_u"], d["W_d"],
                            d["Ws_g"], d["Ws_u"], d["Ws_d"], Y, wsb, cap)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        start.record(stream)
        for i in range(steps):
            if flush is not None:
                flush.fill_(i)   # evict the layer's inputs from L2; outside the step's events
            if graph is not None:
                ev[i][0].record(stream)
                graph.replay()
                ev[i][4].record(stream)
                continue
            moe.moe_set_stage_events(ev[i])
            step(d["x"], Y)
        moe.moe_set_stage_events([])
        end.record(stream)
        torch.cuda.synchronize()
        time.sleep(0.2)
    if ws_n > 1:
        dist.barrier()
    if flush is None:
        ms_total = start.elapsed_time(end)
    else:  # sum of the steps' own spans (first stage event to last)
        ms_total = float(sum(ev[i][0].elapsed_time(ev[i][4]) for i in range(steps)))
    ms_total = max_over_ranks(ms_total, device="cuda")
    ms_step = ms_total / steps
    if graph is not None:
        # stage times from eager steps (a replay records no stage events)
        for i in range(steps):
            moe.moe_set_stage_events(ev[i])
            step(d["x"], Y)
        moe.moe_set_stage_events([])
        torch.cuda.synchronize()
        del graph
    stage_ms = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(4)] for i in range(steps)])
    gate_up_ms = float(stage_ms[:, 2].mean())
    down_ms = float(stage_ms[:, 3].mean())

    # end to end through the public API with host buffers: every step uploads
    # its x from pinned memory, runs the layer and downloads Y to pinned
    # memory; the pipeline overlaps step i's compute with the copies of its
    # neighbours (two device buffers, separate copy streams)
    from sparse_mixture_experts_25_b200.pipeline import HostPipeline
    x_host = torch.from_numpy(np.ascontiguousarray(inp["x"]).view(np.int16)).view(torch.bfloat16) \
        if w.dtype == si.DT_BF16 else torch.from_numpy(inp["x"])
    x_host = x_host.pin_memory()
    y_host = torch.empty(w.N, w.d, dtype=torch.float32).pin_memory()
    fwd = None
    if sharded_group:
        def fwd(xd, yd, wsd, st):
            sharded.forward_sharded(p, N_group, C_group, xd, d["W_r"], d["b_r"], d["lat"], d["W_g"], d["W_u"],
                                    d["W_d"], d["Ws_g"], d["Ws_u"], d["Ws_d"], yd, wsd, counts=counts, stream=st)
    pipe = HostPipeline(p, d, forward=fwd)
    for _ in range(3):
        pipe.submit(x_host, y_host)
    pipe.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws_n > 1:
        dist.barrier()
    e_start.record(pipe.h2d)
    for _ in range(steps):
        pipe.submit(x_host, y_host)
    pipe.compute.wait_stream(pipe.d2h)
    pipe.d2h.wait_stream(pipe.compute)
    e_end.record(pipe.d2h)
    pipe.synchronize()
    e_ms = max_over_ranks(e_start.elapsed_time(e_end), device="cuda") / steps

    peaks, peak_src = load_peaks()
    timed_s = ms_total / 1000.0
    if timed_s < 1.0:
        peak_tf, peak_kind = peaks["bf16_tflops"], "burst"
    else:
        peak_tf, peak_kind = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), "sustained"
    gu_flops = gate_up_flops(w, accepted)
    achieved = gu_flops / (gate_up_ms * 1e-3) / 1e12
    touched = int((moe.workspace_views(p, wsb)["acc"] > 0).sum().item())
    gu_bytes = gate_up_bytes(w, accepted, touched)
    if w.dtype != si.DT_BF16:
        # fp32 layers run the FFMA kernels: bound by CUDA-core arithmetic
        peak_ffma = ffma_peak_tflops(peaks.get("sm_max_mhz", 1965.0))
        roof = {"kernel": "simt_grouped_kernel<SWIGLU> (gate/up GEMM + SwiGLU, fp32 FFMA)",
                "bound": "alu", "achieved": achieved, "peak": peak_ffma, "unit": "TFLOP/s",
                "frac": achieved / peak_ffma, "traffic": None,
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 FLOP x max SM clock"}
    elif gu_bytes / (peaks["hbm_gbs"] * 1e9) > gu_flops / (peak_tf * 1e12):
        # streaming the touched weights takes longer than the MMAs: HBM-bound
        gbs = gu_bytes / (gate_up_ms * 1e-3) / 1e9
        roof = {"kernel": "tc_grouped_kernel<SWIGLU> (gate/up GEMM + SwiGLU)",
                "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"],
                "traffic": committed_traffic("gate_up", w.name),
                "peak_source": f"{peak_src} HBM copy"}
    else:
        roof = {"kernel": "tc_grouped_kernel<SWIGLU> (gate/up GEMM + SwiGLU)",
                "bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved / peak_tf,
                "traffic": committed_traffic("gate_up", w.name),
                "peak_source": f"{peak_src} bf16 {peak_kind}"}
    gu_gbs = gu_bytes / (gate_up_ms * 1e-3) / 1e9
    roof.update({"flops_per_launch": gu_flops, "bytes_per_launch": gu_bytes, "avg_launch_ms": gate_up_ms,
                 "tflops": achieved, "gbs": gu_gbs, "hbm_frac": gu_gbs / peaks["hbm_gbs"]})
    if w.dtype == si.DT_BF16:
        roof["tensor_frac"] = achieved / peak_tf
    line = {
        "metric": METRIC,
        "value": ws_n * w.N / (ms_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": ws_n,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == si.DT_BF16 else "f32",
        "data": "synthetic (seeded SplitMix64/Box-Muller; x~N(0,1), W~N(0,1/fan_in)); no dataset or checkpoint",
        "config": config_of(w, args),
        "roofline": roof,
        "stages_ms": {"route": float(stage_ms[:, 0].mean()), "dispatch": float(stage_ms[:, 1].mean()),
                      "gate_up": gate_up_ms, "down_combine": down_ms},
        "step_tflops": step_flops(w, accepted) / (ms_step * 1e-3) / 1e12,
        "down_tflops": 2.0 * accepted * w.d * w.d_f / (down_ms * 1e-3) / 1e12,
        "e2e": {"value": ws_n * w.N / (e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size()),
                "ms_per_step": e_ms,
                "how": "pinned x upload, moe_forward, pinned Y download per step; copies of "
                       "neighbouring steps overlap compute (HostPipeline, 2 device buffers)"
                       + ("; L2 not flushed between these steps" if flush is not None else "")},
        "gpu_launches": kernels_per_step(w, sharded_group) * steps,
        "clocks": clk.summary(),
        "routing": {k: stats[k] for k in ("accepted", "rejected", "near_tie", "L_max", "rho_max")},
    }
    if cpu_base is not None:
        line["cpu_baseline"] = {k: cpu_base[k] for k in ("value", "unit", "cores", "kind", "sample")}
    return line


def per_config_summary(line: dict) -> dict:
    """The keys of one workload's line that the headline's per_config object carries."""
    keep = ("value", "unit", "ms_per_step", "steps", "warmup", "dtype", "config", "roofline", "stages_ms",
            "e2e", "gpu_launches", "clocks", "routing")
    out = {k: line[k] for k in keep}
    out["roofline"] = {k: line["roofline"][k] for k in ("kernel", "bound", "achieved", "peak", "unit", "frac",
                                                         "traffic", "peak_source", "avg_launch_ms", "hbm_frac")
                       if k in line["roofline"]}
    if "tensor_frac" in line["roofline"]:
        out["roofline"]["tensor_frac"] = line["roofline"]["tensor_frac"]
    out["e2e"] = {k: line["e2e"][k] for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step",
                                              "ms_per_step")}
    return out


def run_gpu(args):
    import torch
    import torch.distributed as dist

    ws_n, rank, local = dist_env()
    w = si.WORKLOADS[args.workload]
    cpu_base = None
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        # the oracle on a bounded sample of the same seeded inputs (host cores,
        # before any CUDA call)
        cpu_base = oracle_sample(w, si.inputs(w), sample_tokens=args.ref_sample)

    torch.cuda.set_device(local)
    if ws_n > 1:
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    line = measure_forward(w, args, args.steps, args.warmup, cpu_base=cpu_base)
    if ws_n == 1 and args.per_config and args.workload == WORKLOAD and not args.graph:
        # the other page-shaped layers, each measured the same way in this run
        per = {}
        for name in PER_CONFIG:
            torch.cuda.empty_cache()
            per[name] = per_config_summary(measure_forward(si.WORKLOADS[name], args, args.steps, args.warmup))
        line["per_config"] = per
        line["gpu_launches"] += sum(v["gpu_launches"] for v in per.values())
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def backward_kernels(w: si.Workload) -> int:
    """Kernels one moe_backward launches: offsets check (1), tables (5), scores
    (1), dY gather (1), z / u / W_d^T dY / dx-row GEMMs (4; W_d, W_g, W_u read
    as stored), SwiGLU backward (1), router (1), router contractions (2, plus
    the slice sum when dW_r = dG^T X is split over the tokens on the CUDA
    cores, or the score split and its tables on the tensor cores), db (2), dx (1),
    row transposes (5), weight-gradient prefixes (2) and GEMMs (3); the shared
    expert adds 19."""
    tiles = ((w.E + 63) // 64) * ((w.d + 63) // 64)
    sms = 148
    slices = max(1, min(-(-2 * sms // tiles), max(1, w.N // 256), 16))
    if w.dtype != si.DT_BF16:
        # fp32: scores, two gathers, SwiGLU, router chain, dx; per touched expert
        # z, u, W_d^T dY, two dx-row and three weight-gradient contractions
        return 1 + 1 + 2 + 1 + (3 + 2 + (1 if slices > 1 else 0)) + 1 + 8 * w.E + (8 if w.d_f_shared else 0)
    # E_r % 64 == 0: the router contractions run on the tensor cores, after a
    # score split and a table kernel (no slice sum)
    router_tc = w.E % 64 == 0 and w.N % 8 == 0
    return 29 + (2 if router_tc else (1 if slices > 1 else 0)) + (19 if w.d_f_shared else 0)


def run_gpu_backward(args):
    """--backward: one GPU; the forward runs once (routing records, x_perm,
    h), then moe_backward is timed: gradients of sum(dY * Y) + 0.01 aux with
    respect to x, W_r, b_r, the experts and the shared expert."""
    import torch
    import sparse_mixture_experts_25_b200 as moe
    if dist_env()[0] > 1:
        raise SystemExit("--backward runs on one GPU")
    w = si.WORKLOADS[args.workload]
    inp = si.inputs(w)
    dY_host = si.upstream_gradient(w)
    torch.cuda.set_device(0)

    def dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    d = {k: dev(v) for k, v in inp.items()}
    p = moe.params(w.N, w.d, w.d_f, w.E, w.k, c=w.c, norm=w.norm, theta=w.theta, dtype=w.dtype,
                   d_f_shared=w.d_f_shared, reject_policy=w.reject_policy, accept_order=w.accept_order)
    wsb = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    Y = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    moe.moe_forward(p, d["x"], d["W_r"], d["b_r"], d["lat"], d["W_g"], d["W_u"], d["W_d"], d["Ws_g"], d["Ws_u"],
                    d["Ws_d"], Y, wsb)
    status, stats = moe.moe_get_stats(p, wsb)
    if status != moe.MOE_OK:
        raise RuntimeError(f"moe_forward status: {moe.moe_status_string(status)}")
    offsets = moe.workspace_views(p, wsb)["offsets"].cpu().numpy()
    dY = torch.from_numpy(dY_host).cuda()
    shapes = {"dx": (w.N, w.d), "dW_r": (w.E, w.d), "db_r": (w.E,), "dW_g": (w.E, w.d_f, w.d),
              "dW_u": (w.E, w.d_f, w.d), "dW_d": (w.E, w.d, w.d_f)}
    if w.d_f_shared:
        shapes.update({"dWs_g": (w.d_f_shared, w.d), "dWs_u": (w.d_f_shared, w.d), "dWs_d": (w.d, w.d_f_shared)})
    g = {n: torch.empty(sh, dtype=torch.float32, device="cuda") for n, sh in shapes.items()}
    bws = torch.empty(moe.moe_backward_workspace_size(p, offsets), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        moe.moe_backward(p, offsets, d["x"], d["W_r"], d["b_r"], d["W_g"], d["W_u"], d["W_d"], d["Ws_g"],
                         d["Ws_u"], d["Ws_d"], dY, wsb, g, bws, aux_coef=0.01, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if moe.moe_backward_check(p, bws) != moe.MOE_OK:
        raise RuntimeError("moe_backward: a bounded device wait timed out")
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.int32, device="cuda")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(0) as clk:
        time.sleep(0.3)
        for i in range(args.steps):
            flush.fill_(i)   # evict the layer's data from L2; outside the step's events
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        time.sleep(0.2)
    ms_step = float(sum(a.elapsed_time(b) for a, b in ev)) / args.steps
    R = int(stats["accepted"])
    touched = int((moe.workspace_views(p, wsb)["acc"] > 0).sum().item())
    ds = w.d_f_shared
    # 8 contractions of the expert size per routed row: z, u (recomputed), W_d^T dY,
    # dx rows (two), dW_d, dW_g, dW_u; the same over every token for the shared
    # expert; the router's three E_r-wide contractions
    flops = 16.0 * R * w.d * w.d_f + 16.0 * w.N * w.d * ds + 6.0 * w.N * w.E * w.d
    # least HBM traffic: bf16 weights read, fp32 weight gradients written, x and
    # dY read, dx written
    es = 2 if w.dtype == si.DT_BF16 else 4
    nbytes = (3.0 * touched * w.d * w.d_f * (es + 4) + 3.0 * w.d * ds * (es + 4)
              + w.N * w.d * (es + 4 + 4) + w.E * w.d * (es + 4))
    peaks, peak_src = load_peaks()
    timed_s = ms_step * args.steps / 1000.0
    peak_tf = peaks["bf16_tflops"] if timed_s < 1.0 else peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    t_tensor = flops / (peak_tf * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    tflops = flops / (ms_step * 1e-3) / 1e12
    gbs = nbytes / (ms_step * 1e-3) / 1e9
    if w.dtype != si.DT_BF16:
        # fp32 layers contract on the CUDA cores: bound by FP32 arithmetic
        peak_ffma = ffma_peak_tflops(peaks.get("sm_max_mhz", 1965.0))
        roof = {"bound": "alu", "achieved": tflops, "peak": peak_ffma, "unit": "TFLOP/s",
                "frac": tflops / peak_ffma}
    elif t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": tflops, "peak": peak_tf, "unit": "TFLOP/s", "frac": tflops / peak_tf}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    roof.update({"kernel": "moe_backward, all launches of one call", "traffic": None,
                 "flops_per_launch": flops, "bytes_per_launch": nbytes, "avg_launch_ms": ms_step,
                 "peak_source": f"{peak_src} bf16 {'burst' if timed_s < 1.0 else 'sustained'} / HBM copy"})
    line = {
        "metric": "MoE-layer backward tokens/s (gradients of x, W_r, b_r, experts, shared expert)",
        "value": w.N / (ms_step * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == si.DT_BF16 else "f32",
        "data": "synthetic (seeded; dY ~ N(0,1)); no dataset or checkpoint",
        "config": dict(config_of(w, args), l2="flushed between steps (256 MiB write)"),
        "roofline": roof, "gpu_launches": backward_kernels(w) * args.steps, "clocks": clk.summary(),
        "routing": {k: stats[k] for k in ("accepted", "rejected", "L_max")},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(si.WORKLOADS))
    ap.add_argument("--ref-sample", type=int, default=32)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-config", dest="per_config", action="store_true", default=True,
                    help="with the default workload on one GPU, also measure the other page-shaped layers "
                         "(per_config object; default on)")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of one step captured into a CUDA graph (one GPU)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (one GPU, bf16 layers) instead of the forward")
    ap.add_argument("--override", action="append", default=[],
                    help="key=value change of the workload shape (profiling of smaller cases)")
    args = ap.parse_args(argv)
    if args.override:
        w = si.WORKLOADS[args.workload]
        kw = {}
        for item in args.override:
            key, val = item.split("=", 1)
            kw[key] = type(getattr(w, key))(val)
        name = w.name + "[" + ",".join(args.override) + "]"
        si.WORKLOADS[name] = w.scaled(name, **kw)
        args.workload = name
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.backward:
        return run_gpu_backward(args)
    if si.WORKLOADS[args.workload].soft_p > 0:
        return run_gpu_soft(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
