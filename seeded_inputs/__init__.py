"""Seeded synthetic inputs for the sparse-MoE layer: the one module that the CPU
oracle and the CUDA path both read.

It holds random-number generation and the workload table only; none of the
layer's arithmetic (routing, capacity, experts, combine) lives here.  Every
element is a pure function of (seed, tensor id, index), computed by the C
generator in ``gen.c`` (SplitMix64 + Box-Muller); ``reference_normals`` is an
independent numpy restatement of the same published definitions, used by the
tests to pin the C code.

Workloads follow the five layer shapes of the source pages (a Switch-style
top-1 layer, a Mixtral-shaped layer, a Qwen3-235B-shaped layer with skewed
routing, a DeepSeek-V3-shaped layer with a shared expert, and a WDMoE decode
batch with weight-latency-ratio pruning), plus scaled-down variants built
with the same recipe for fast parity tests.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libseeded.so")

NORM_RENORM, NORM_FULLPROB, NORM_WLR = 0, 1, 2
DT_F32, DT_BF16 = 0, 1

# tensor ids of the counter-based streams
TID = {"x": 1, "W_r": 2, "W_g": 3, "W_u": 4, "W_d": 5, "Ws_g": 6, "Ws_u": 7, "Ws_d": 8,
       "lat_up": 9, "lat_comp": 10, "lat_down": 11, "Phi": 12, "dY": 13}


def build(force: bool = False) -> str:
    """Compile gen.c into libseeded.so beside it (gcc, -O2, pthreads)."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
                               "-o", tmp, src, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.sg_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                ctypes.c_void_p, ctypes.c_int]
        lib.sg_fill.restype = ctypes.c_int
        lib.sg_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                               ctypes.c_void_p]
        lib.sg_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.sg_stream_key.restype = ctypes.c_uint64
        _lib = lib
    return _lib


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def fill(seed: int, tensor_id: int, count: int, *, start: int = 0, kind: str = "normal",
         mean: float = 0.0, std: float = 1.0, dtype: str = "f32") -> np.ndarray:
    """Elements [start, start+count) of one stream.  dtype 'f32', 'bf16'
    (returned as uint16 bit patterns) or 'f64'; kind 'normal' or 'lognormal'."""
    lib = _load()
    np_dt = {"f32": np.float32, "bf16": np.uint16, "f64": np.float64}[dtype]
    code = {"f32": 0, "bf16": 1, "f64": 2}[dtype]
    out = np.empty(count, dtype=np_dt)
    if count:
        lib.sg_fill(seed, tensor_id, start, count, 0 if kind == "normal" else 1, mean, std, code,
                    out.ctypes.data, host_threads())
    return out


def raw_u64(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    lib = _load()
    out = np.empty(count, dtype=np.uint64)
    lib.sg_u64(seed, tensor_id, start, count, out.ctypes.data)
    return out


# ---------------------------------------------------------------------------
# Independent numpy restatement (used only to pin the C generator in tests)
# ---------------------------------------------------------------------------
_M = np.uint64(0xFFFFFFFFFFFFFFFF)


def _mix64_np(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def reference_u64(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    gamma = np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        s = _mix64_np(np.array([np.uint64(seed) + gamma], dtype=np.uint64))[0]
        key = _mix64_np(np.array([s ^ (np.uint64(tensor_id) * np.uint64(0xD1B54A32D192ED03))],
                                 dtype=np.uint64))[0]
        i = np.arange(start, start + count, dtype=np.uint64)
        return _mix64_np(key + (i + np.uint64(1)) * gamma)


def reference_normals(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """Box-Muller standard normals in float64, restated with numpy."""
    idx = np.arange(start, start + count, dtype=np.int64)
    j = idx // 2
    lo, hi = int(j.min()) * 2, int(j.max()) * 2 + 2
    u = reference_u64(seed, tensor_id, lo, hi - lo)
    a = u[(2 * j - lo)]
    b = u[(2 * j + 1 - lo)]
    u1 = ((a >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * 2.0 ** -53
    u2 = (b >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    r = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    return np.where(idx % 2 == 1, r * np.sin(ang), r * np.cos(ang))


# ---------------------------------------------------------------------------
# bf16 helpers (storage format only)
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    nan = (u & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    r[nan] = ((u[nan] >> np.uint32(16)) | np.uint32(0x40)).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    d: int
    d_f: int
    E: int
    k: int
    norm: int = NORM_RENORM
    c: float = 0.0              # capacity factor; <= 0 means no capacity limit
    theta: float = 0.0          # WLR threshold (NORM_WLR only)
    dtype: int = DT_BF16
    d_f_shared: int = 0         # 0 = no shared expert
    zipf_s: float = 0.0         # > 0: router bias b_e = 0.5 ln(Zipf(s) weight of rank e+1)
    latency: bool = False       # per-token per-expert latency t = t_up + t_comp + t_down
    seed: int = 25000
    reject_policy: int = 0      # 0: rejected path adds 0; 1: accepted paths renormalised; 2: rerouted
    accept_order: int = 0       # 0: token order; 1: largest routing weight first
    reroute_depth: int = 0      # reject_policy 2: next-ranked experts a token may try
    soft_p: int = 0             # > 0: Soft MoE layer with soft_p slots per expert (Phi [E soft_p, d])

    @property
    def dt(self) -> str:
        return "bf16" if self.dtype == DT_BF16 else "f32"

    def scaled(self, name: str, **kw) -> "Workload":
        return dataclasses.replace(self, name=name, **kw)


WORKLOADS = {
    "switch_top1_f32": Workload("switch_top1_f32", N=1024, d=256, d_f=512, E=8, k=1,
                                norm=NORM_FULLPROB, c=1.25, dtype=DT_F32, seed=25000),
    "mixtral_bf16": Workload("mixtral_bf16", N=4096, d=4096, d_f=14336, E=8, k=2,
                             norm=NORM_RENORM, seed=25001),
    "qwen3_skew_bf16": Workload("qwen3_skew_bf16", N=8192, d=4096, d_f=1536, E=128, k=8,
                                norm=NORM_RENORM, c=1.25, zipf_s=1.2, seed=25002),
    "deepseek_shared_bf16": Workload("deepseek_shared_bf16", N=4096, d=7168, d_f=2048, E=256, k=8,
                                     norm=NORM_RENORM, d_f_shared=2048, seed=25003),
    "wdmoe_decode_bf16": Workload("wdmoe_decode_bf16", N=64, d=4096, d_f=14336, E=8, k=2,
                                  norm=NORM_WLR, theta=0.3, latency=True, seed=25004),
    # routing variants on the Mixtral shape (the pages give no configuration for them):
    # expert choice with C = N k / E_r for k = 2, and Soft MoE with S = N slots
    "expert_choice_bf16": Workload("expert_choice_bf16", N=4096, d=4096, d_f=14336, E=8, k=8,
                                   norm=NORM_FULLPROB, c=0.25, accept_order=1, seed=25005),
    "soft_moe_bf16": Workload("soft_moe_bf16", N=4096, d=4096, d_f=14336, E=8, k=1, soft_p=512,
                              seed=25006),
}


def shape(w: Workload, name: str):
    return {
        "x": (w.N, w.d), "W_r": (w.E, w.d), "b_r": (w.E,), "lat": (w.N, w.E),
        "W_g": (w.E, w.d_f, w.d), "W_u": (w.E, w.d_f, w.d), "W_d": (w.E, w.d, w.d_f),
        "Ws_g": (w.d_f_shared, w.d), "Ws_u": (w.d_f_shared, w.d), "Ws_d": (w.d, w.d_f_shared),
        "Phi": (w.E * w.soft_p, w.d),
    }[name]


def _std(w: Workload, name: str) -> float:
    if name in ("x",):
        return 1.0
    if name in ("W_r", "W_g", "W_u", "Ws_g", "Ws_u", "Phi"):
        return 1.0 / math.sqrt(w.d)
    if name == "W_d":
        return 1.0 / math.sqrt(w.d_f)
    if name == "Ws_d":
        return 1.0 / math.sqrt(w.d_f_shared)
    raise KeyError(name)


def tensor(w: Workload, name: str, expert: Optional[int] = None) -> Optional[np.ndarray]:
    """Host copy of one input tensor of workload w (None where the workload has
    no such input).  Floating tensors come in the workload's storage dtype
    (bf16 as uint16 bits); b_r and lat are always fp32.  For the per-expert
    weights, ``expert`` selects one expert's [out, in] slice."""
    if name == "b_r":
        if w.zipf_s <= 0:
            return None
        r = np.arange(1, w.E + 1, dtype=np.float64)
        p = r ** (-w.zipf_s)
        p /= p.sum()
        return (0.5 * np.log(p)).astype(np.float32)
    if name == "lat":
        if not w.latency:
            return None
        n = w.N * w.E
        t = sum(fill(w.seed, TID[part], n, kind="lognormal", mean=0.0, std=0.5, dtype="f64")
                for part in ("lat_up", "lat_comp", "lat_down"))
        return t.astype(np.float32).reshape(w.N, w.E)
    if name.startswith("Ws_") and w.d_f_shared <= 0:
        return None
    if name == "Phi" and w.soft_p <= 0:
        return None
    shp = shape(w, name)
    if expert is not None:
        assert name in ("W_g", "W_u", "W_d")
        per = shp[1] * shp[2]
        a = fill(w.seed, TID[name], per, start=expert * per, std=_std(w, name), dtype=w.dt)
        return a.reshape(shp[1], shp[2])
    n = int(np.prod(shp))
    return fill(w.seed, TID[name], n, std=_std(w, name), dtype=w.dt).reshape(shp)


def upstream_gradient(w: Workload, seed_offset: int = 0) -> np.ndarray:
    """The gradient dL/dY [N, d] fed to the layer's backward pass: standard
    normals in fp32 (the backward rounds it to its own precision)."""
    n = w.N * w.d
    return fill(w.seed + seed_offset, TID["dY"], n, std=1.0, dtype="f32").reshape(w.N, w.d)


def inputs(w: Workload, names=("x", "W_r", "b_r", "lat", "W_g", "W_u", "W_d", "Ws_g", "Ws_u", "Ws_d")):
    return {n: tensor(w, n) for n in names}
