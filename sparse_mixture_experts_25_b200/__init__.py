"""Python binding of libmoe, the B200 (sm_100a) sparse-MoE layer forward pass.

Argument marshalling only: every function here passes device pointers of
torch tensors (torch is used for device memory and streams) and the current
CUDA stream to the C ABI declared in include/moe.h, under the same names.
All computation runs in the library's CUDA kernels.  There is no fallback:
if libmoe.so cannot be built or loaded, importing this package fails.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

from . import build as _build

__all__ = [
    "MoEError", "Params", "Stats", "WsLayout", "lib", "params", "moe_capacity",
    "moe_workspace_size", "moe_workspace_layout", "moe_route", "moe_dispatch",
    "moe_dispatch_noalloc",
    "moe_expert_ffn", "moe_combine", "moe_forward", "moe_forward_begin", "moe_forward_end",
    "moe_get_stats",
    "moe_set_stage_events", "moe_selftest_wait_timeout", "moe_status_string", "moe_last_error",
    "expert_choice_params", "SoftParams", "soft_params", "moe_soft_workspace_size", "moe_soft_forward",
    "moe_dispatch_ranked", "moe_gather_rows", "workspace_x_perm",
    "moe_ep_plan", "moe_ep_dispatch", "moe_ep_combine", "pointer_table",
    "moe_soft_check",
    "workspace_views", "HEADER",
]

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_NONFINITE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_WORKSPACE, MOE_ERR_TIMEOUT = 4, 5, 6
MOE_NORM_RENORM, MOE_NORM_FULLPROB, MOE_NORM_WLR = 0, 1, 2
MOE_F32, MOE_BF16 = 0, 1
MOE_REJECT_ZERO, MOE_REJECT_RENORM, MOE_REJECT_REROUTE = 0, 1, 2
MOE_ACCEPT_TOKEN, MOE_ACCEPT_WEIGHT = 0, 1

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status in (MOE_ERR_CUDA, MOE_ERR_UNSUPPORTED) and moe_last_error():
            detail = f" [{moe_last_error()}]"
        super().__init__(f"{where}: {moe_status_string(status)} (status {status}){detail}")


class Params(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("d", ctypes.c_int32), ("d_f", ctypes.c_int32),
                ("E_r", ctypes.c_int32), ("k", ctypes.c_int32), ("c", ctypes.c_double),
                ("norm", ctypes.c_int32), ("theta", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("d_f_shared", ctypes.c_int32), ("reject_policy", ctypes.c_int32),
                ("accept_order", ctypes.c_int32), ("reroute_depth", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class SoftParams(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("d", ctypes.c_int32), ("d_f", ctypes.c_int32),
                ("E_r", ctypes.c_int32), ("p", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


def soft_params(N, d, d_f, E_r, p, dtype=None) -> SoftParams:
    """Soft MoE layer: S = E_r p slots (see moe_soft_forward in the header)."""
    return SoftParams(int(N), int(d), int(d_f), int(E_r), int(p), int(MOE_BF16 if dtype is None else dtype), 0)


class Stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "C", "requested", "accepted", "rejected", "O", "tokens_affected", "tokens_skipped",
        "nonfinite", "near_tie", "L_max", "L_p50", "L_p90", "L_p99")] + [
        ("rho_max", ctypes.c_double), ("reject_rate", ctypes.c_double),
        ("device_error", ctypes.c_int32), ("rerouted", ctypes.c_int32),
        ("padded_rows", ctypes.c_int64), ("padding_ratio", ctypes.c_double),
        ("aux_balance", ctypes.c_double)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_LAYOUT_FIELDS = ("ids", "w", "margin", "slot", "offsets", "L", "acc", "slot_token", "slot_w",
                  "counters", "x_perm", "h", "h_shared", "cand", "cand_w", "rr_e", "rr_slot", "scratch", "total")


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in _LAYOUT_FIELDS]


_P = ctypes.c_void_p
_lib = None


GRAD_NAMES = ("dx", "dW_r", "db_r", "dW_g", "dW_u", "dW_d", "dWs_g", "dWs_u", "dWs_d")


class Grads(ctypes.Structure):
    """moe_grads: device pointers of the gradient buffers (fp32)."""
    _fields_ = [(n, _P) for n in GRAD_NAMES]


def lib():
    """Load (building first if missing or stale) the in-tree libmoe.so, or the
    library file named by the MOE_LIB_PATH environment variable."""
    global _lib
    if _lib is None:
        path = os.environ.get("MOE_LIB_PATH") or _build.build()
        L = ctypes.CDLL(path)
        pp = ctypes.POINTER(Params)
        L.moe_capacity.argtypes = [pp, ctypes.POINTER(ctypes.c_int64)]
        L.moe_workspace_size.argtypes = [pp, ctypes.POINTER(ctypes.c_size_t)]
        L.moe_workspace_layout.argtypes = [pp, ctypes.POINTER(WsLayout)]
        L.moe_route.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        L.moe_dispatch.argtypes = [pp, _P, _P, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P]
        L.moe_dispatch_noalloc.argtypes = [pp, _P, _P, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P]
        L.moe_expert_ffn.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P]
        L.moe_combine.argtypes = [pp, _P, _P, _P, _P, _P, _P]
        L.moe_forward.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        L.moe_get_stats.argtypes = [pp, _P, ctypes.POINTER(Stats), _P]
        L.moe_forward_begin.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P]
        L.moe_forward_end.argtypes = [pp, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                      ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        L.moe_set_stage_events.argtypes = [ctypes.POINTER(_P), ctypes.c_int]
        L.moe_selftest_wait_timeout.argtypes = [pp, _P, ctypes.c_int64, _P]
        L.moe_dispatch_ranked.argtypes = [pp, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                          ctypes.c_int64, _P, _P, _P]
        L.moe_gather_rows.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int64, _P, _P]
        L.moe_ep_plan.argtypes = [pp, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P]
        L.moe_ep_dispatch.argtypes = [pp, ctypes.c_int32, _P, _P, _P, _P]
        L.moe_ep_combine.argtypes = [pp, ctypes.c_int32, _P, _P, _P, _P]
        sp = ctypes.POINTER(SoftParams)
        L.moe_soft_workspace_size.argtypes = [sp, ctypes.POINTER(ctypes.c_size_t)]
        L.moe_soft_forward.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P, _P]
        L.moe_soft_check.argtypes = [sp, _P, _P]
        L.moe_backward_workspace_size.argtypes = [pp, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_size_t)]
        L.moe_backward.argtypes = [pp, ctypes.c_float, ctypes.POINTER(ctypes.c_int32), _P, _P, _P, _P, _P, _P,
                                   _P, _P, _P, _P, _P, ctypes.POINTER(Grads), _P, ctypes.c_size_t, _P]
        L.moe_backward_check.argtypes = [pp, _P, _P]
        L.moe_last_error.argtypes = []
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        for name in ("moe_capacity", "moe_workspace_size", "moe_workspace_layout", "moe_route",
                     "moe_dispatch", "moe_dispatch_noalloc", "moe_expert_ffn", "moe_combine",
                     "moe_forward",
                     "moe_get_stats", "moe_set_stage_events", "moe_forward_begin",
                     "moe_forward_end", "moe_selftest_wait_timeout", "moe_soft_workspace_size",
                     "moe_soft_forward", "moe_soft_check", "moe_dispatch_ranked", "moe_gather_rows",
                     "moe_backward_workspace_size", "moe_backward", "moe_backward_check"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def declared_symbols():
    """Entry points declared in include/moe.h."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, flags=re.M)))


def params(N, d, d_f, E_r, k, c=0.0, norm=MOE_NORM_RENORM, theta=0.0, dtype=MOE_BF16,
           d_f_shared=0, reject_policy=MOE_REJECT_ZERO, accept_order=MOE_ACCEPT_TOKEN,
           reroute_depth=0) -> Params:
    """moe_params; reroute_depth is the number of next-ranked experts a token
    may try under MOE_REJECT_REROUTE (ignored by the other policies)."""
    return Params(int(N), int(d), int(d_f), int(E_r), int(k), float(c), int(norm), float(theta),
                  int(dtype), int(d_f_shared), int(reject_policy), int(accept_order), int(reroute_depth), 0)


def expert_choice_params(N, d, d_f, E_r, C, dtype=MOE_BF16, d_f_shared=0) -> Params:
    """Parameters under which moe_forward computes expert-choice routing: every
    token requests every expert (k = E_r) with its full-softmax probability as
    the weight, and each expert accepts the C requests with the largest weight
    (acceptance by weight), i.e. picks its C tokens by its score column.  The
    capacity C = ceil(c N k / E_r) = ceil(c N) is reached with c = C / N.
    E_r <= 32 (the library's limit on k)."""
    if not (1 <= int(C) <= max(int(N), 1)):
        raise ValueError("expert choice needs 1 <= C <= N")
    return params(N, d, d_f, E_r, E_r, c=float(C) / max(int(N), 1), norm=MOE_NORM_FULLPROB, dtype=dtype,
                  d_f_shared=d_f_shared, accept_order=MOE_ACCEPT_WEIGHT)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libmoe takes device tensors; got a host tensor")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def moe_last_error() -> str:
    return lib().moe_last_error().decode()


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def moe_capacity(p: Params) -> int:
    C = ctypes.c_int64()
    _check(lib().moe_capacity(ctypes.byref(p), ctypes.byref(C)), "moe_capacity")
    return C.value


def moe_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check(lib().moe_workspace_size(ctypes.byref(p), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_workspace_layout(p: Params) -> dict:
    L = WsLayout()
    _check(lib().moe_workspace_layout(ctypes.byref(p), ctypes.byref(L)), "moe_workspace_layout")
    return {n: getattr(L, n) for n in _LAYOUT_FIELDS}


def moe_route(p, x, W_r, b_r, lat, ids, w, margin, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(p), _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(lat), _ptr(ids),
                           _ptr(w), _ptr(margin), _ptr(ws), _stream(stream)), "moe_route")


def moe_dispatch(p, ids, w, C, slot, offsets, slot_token, slot_w, x, x_perm, ws, stream=None):
    _check(lib().moe_dispatch(ctypes.byref(p), _ptr(ids), _ptr(w), int(C), _ptr(slot), _ptr(offsets),
                              _ptr(slot_token), _ptr(slot_w), _ptr(x), _ptr(x_perm), _ptr(ws),
                              _stream(stream)), "moe_dispatch")


def moe_dispatch_noalloc(p, ids, w, C, slot, offsets, slot_token, slot_w, x, x_perm, stream=None):
    """moe_dispatch with its scratch in the library's static device buffer
    (for callers that cannot allocate device memory at the call site)."""
    _check(lib().moe_dispatch_noalloc(ctypes.byref(p), _ptr(ids), _ptr(w), int(C), _ptr(slot),
                                      _ptr(offsets), _ptr(slot_token), _ptr(slot_w), _ptr(x),
                                      _ptr(x_perm), _stream(stream)), "moe_dispatch_noalloc")


def moe_expert_ffn(p, x_perm, offsets, W_g, W_u, W_d, H, ws, stream=None):
    _check(lib().moe_expert_ffn(ctypes.byref(p), _ptr(x_perm), _ptr(offsets), _ptr(W_g), _ptr(W_u),
                                _ptr(W_d), _ptr(H), _ptr(ws), _stream(stream)), "moe_expert_ffn")


def moe_combine(p, H, offsets, slot_token, slot_w, Y, stream=None):
    _check(lib().moe_combine(ctypes.byref(p), _ptr(H), _ptr(offsets), _ptr(slot_token), _ptr(slot_w),
                             _ptr(Y), _stream(stream)), "moe_combine")


def moe_forward(p, x, W_r, b_r, lat, W_g, W_u, W_d, Ws_g, Ws_u, Ws_d, Y, ws, stream=None):
    _check(lib().moe_forward(ctypes.byref(p), _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(lat), _ptr(W_g),
                             _ptr(W_u), _ptr(W_d), _ptr(Ws_g), _ptr(Ws_u), _ptr(Ws_d), _ptr(Y),
                             _ptr(ws), _stream(stream)), "moe_forward")


def moe_forward_begin(p, x, W_r, b_r, lat, counts, ws, stream=None):
    _check(lib().moe_forward_begin(ctypes.byref(p), _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(lat),
                                   _ptr(counts), _ptr(ws), _stream(stream)), "moe_forward_begin")


def moe_forward_end(p, counts_all, rank, n_ranks, N_group, C, x, W_g, W_u, W_d, Ws_g, Ws_u, Ws_d, Y, ws,
                    stream=None):
    _check(lib().moe_forward_end(ctypes.byref(p), _ptr(counts_all), int(rank), int(n_ranks),
                                 int(N_group), int(C), _ptr(x), _ptr(W_g), _ptr(W_u), _ptr(W_d),
                                 _ptr(Ws_g), _ptr(Ws_u), _ptr(Ws_d), _ptr(Y), _ptr(ws),
                                 _stream(stream)), "moe_forward_end")


def moe_get_stats(p, ws, stream=None):
    """Returns (status, stats dict); waits for the stream."""
    s = Stats()
    status = lib().moe_get_stats(ctypes.byref(p), _ptr(ws), ctypes.byref(s), _stream(stream))
    if status not in (MOE_OK, MOE_ERR_NONFINITE, MOE_ERR_TIMEOUT):
        raise MoEError(status, "moe_get_stats")
    return status, s.as_dict()


def moe_dispatch_ranked(p, counts_all, rank: int, n_ranks: int, N_group: int, C: int, x, ws, stream=None):
    """Dispatch of a sharded routing group into the workspace (after
    moe_forward_begin and the count exchange)."""
    _check(lib().moe_dispatch_ranked(ctypes.byref(p), _ptr(counts_all), int(rank), int(n_ranks), int(N_group),
                                     int(C), _ptr(x), _ptr(ws), _stream(stream)), "moe_dispatch_ranked")


def moe_ep_plan(p, counts_all, rank: int, n_ranks: int, C: int, local_offsets, send_rows, recv_rows, ws,
                regroup=None, regroup_inv=None, stream=None):
    """Plan of an expert-parallel step from the exchanged counts (device
    tensors; see moe_ep_plan in include/moe.h)."""
    _check(lib().moe_ep_plan(ctypes.byref(p), _ptr(counts_all), int(rank), int(n_ranks), int(C), _ptr(local_offsets),
                             _ptr(send_rows), _ptr(recv_rows), _ptr(regroup), _ptr(regroup_inv), _ptr(ws),
                             _stream(stream)), "moe_ep_plan")


def pointer_table(buffers, device="cuda"):
    """A device int64 tensor holding the device addresses of `buffers`
    (tensors or integer addresses), for moe_ep_dispatch / moe_ep_combine."""
    import torch
    addrs = [b if isinstance(b, int) else b.data_ptr() for b in buffers]
    return torch.tensor(addrs, dtype=torch.int64, device=device)


def moe_ep_dispatch(p, n_ranks: int, x, recv_table, ws, stream=None):
    """This rank's accepted rows of x into their owners' buffers (recv_table:
    pointer_table of the ranks' receive buffers)."""
    _check(lib().moe_ep_dispatch(ctypes.byref(p), int(n_ranks), _ptr(x), _ptr(recv_table), _ptr(ws),
                                 _stream(stream)), "moe_ep_dispatch")


def moe_ep_combine(p, n_ranks: int, out_table, Y, ws, stream=None):
    """Y += weighted expert outputs read from their owners' output buffers
    (out_table: pointer_table of the ranks' fp32 output buffers)."""
    _check(lib().moe_ep_combine(ctypes.byref(p), int(n_ranks), _ptr(out_table), _ptr(Y), _ptr(ws),
                                _stream(stream)), "moe_ep_combine")


def moe_gather_rows(src, index, dst, stream=None):
    """dst[i] = src[index[i]] for the rows of index (device tensors)."""
    n = int(index.numel())
    row_bytes = src[0].numel() * src.element_size() if src.dim() > 1 else src.element_size()
    _check(lib().moe_gather_rows(_ptr(src), _ptr(index), n, int(row_bytes), _ptr(dst), _stream(stream)),
           "moe_gather_rows")


def moe_soft_workspace_size(sp) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_soft_workspace_size(ctypes.byref(sp), ctypes.byref(n)), "moe_soft_workspace_size")
    return n.value


def moe_soft_forward(sp, x, Phi, W_g, W_u, W_d, Y, ws, stream=None):
    """Soft MoE forward on device tensors (asynchronous)."""
    _check(lib().moe_soft_forward(ctypes.byref(sp), _ptr(x), _ptr(Phi), _ptr(W_g), _ptr(W_u), _ptr(W_d),
                                  _ptr(Y), _ptr(ws), _stream(stream)), "moe_soft_forward")


def moe_soft_check(sp, ws, stream=None) -> int:
    """Waits for the stream; MOE_OK or MOE_ERR_TIMEOUT."""
    return lib().moe_soft_check(ctypes.byref(sp), _ptr(ws), _stream(stream))


def moe_selftest_wait_timeout(p, ws, limit_ns: int, stream=None):
    """Run the bounded-wait self-test into ws's counters (see the header);
    moe_get_stats afterwards reports MOE_ERR_TIMEOUT."""
    _check(lib().moe_selftest_wait_timeout(ctypes.byref(p), _ptr(ws), int(limit_ns), _stream(stream)),
           "moe_selftest_wait_timeout")


def moe_set_stage_events(events):
    """events: list of torch.cuda.Event(enable_timing=True) (>= 5) or [] to stop.
    torch creates the underlying CUDA event on its first record, so an event
    without one is recorded once here to create it."""
    n = len(events)
    for e in events:
        if not e.cuda_event:
            e.record()
    arr = (_P * max(n, 1))(*[e.cuda_event for e in events])
    _check(lib().moe_set_stage_events(arr if n else None, n), "moe_set_stage_events")


def workspace_views(p: Params, ws):
    """Typed torch views of the routing records inside a workspace tensor."""
    import torch
    L = moe_workspace_layout(p)
    N, k, E = p.N, p.k, p.E_r

    def view(name, count, dtype, shape):
        nbytes = count * torch.empty((), dtype=dtype).element_size()
        return ws[L[name]:L[name] + nbytes].view(dtype).view(*shape)

    out = {
        "ids": view("ids", N * k, torch.int32, (N, k)),
        "w": view("w", N * k, torch.float32, (N, k)),
        "margin": view("margin", N, torch.float32, (N,)),
        "slot": view("slot", N * k, torch.int32, (N, k)),
        "offsets": view("offsets", E + 1, torch.int32, (E + 1,)),
        "L": view("L", E, torch.int32, (E,)),
        "acc": view("acc", E, torch.int32, (E,)),
        "slot_token": view("slot_token", N * k, torch.int32, (N * k,)),
        "slot_w": view("slot_w", N * k, torch.float32, (N * k,)),
    }
    if p.reject_policy == MOE_REJECT_REROUTE:
        X = p.reroute_depth
        out.update({
            "cand": view("cand", N * X, torch.int32, (N, X)),
            "cand_w": view("cand_w", N * X, torch.float32, (N, X)),
            "rr_e": view("rr_e", N * k, torch.int32, (N, k)),
            "rr_slot": view("rr_slot", N * k, torch.int32, (N, k)),
        })
    return out


def workspace_x_perm(p: Params, ws):
    """The gathered rows x_perm [N k, d] inside a workspace tensor (accepted
    rows first, grouped by expert as offsets says)."""
    import torch
    L = moe_workspace_layout(p)
    dt = torch.bfloat16 if p.dtype == MOE_BF16 else torch.float32
    n = p.N * p.k * p.d
    nbytes = n * torch.empty((), dtype=dt).element_size()
    return ws[L["x_perm"]:L["x_perm"] + nbytes].view(dt).view(p.N * p.k, p.d)


def _offsets_arg(p, offsets_host):
    import numpy as np
    off = np.ascontiguousarray(np.asarray(offsets_host), dtype=np.int32)
    if off.shape != (p.E_r + 1,):
        raise ValueError("offsets_host must hold E_r + 1 entries")
    return off


def moe_backward_workspace_size(p: Params, offsets_host=None) -> int:
    """Backward workspace bytes for the forward's offsets (host array), or
    the bound for any routing when offsets_host is None."""
    n = ctypes.c_size_t()
    off = None if offsets_host is None else _offsets_arg(p, offsets_host)
    ptr = None if off is None else off.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    _check(lib().moe_backward_workspace_size(ctypes.byref(p), ptr, ctypes.byref(n)), "moe_backward_workspace_size")
    return n.value


def moe_backward(p, offsets_host, x, W_r, b_r, W_g, W_u, W_d, Ws_g, Ws_u, Ws_d, dY, ws, grads, bws,
                 aux_coef: float = 0.0, stream=None):
    """Gradients of sum(dY * Y) + aux_coef * aux for the forward last run on
    ws (see moe_backward in include/moe.h).  offsets_host: the forward's
    offsets [E_r + 1] on the host (a numpy array or CPU tensor); grads: dict
    of device fp32 tensors keyed by GRAD_NAMES (db_r and the shared-expert
    entries may be missing or None); bws: a uint8 device tensor of at least
    moe_backward_workspace_size(p, offsets_host) bytes."""
    off = _offsets_arg(p, offsets_host)
    g = Grads(*[_ptr(grads.get(n)) for n in GRAD_NAMES])
    _check(lib().moe_backward(ctypes.byref(p), float(aux_coef), off.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                              _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(W_g), _ptr(W_u), _ptr(W_d), _ptr(Ws_g), _ptr(Ws_u),
                              _ptr(Ws_d), _ptr(dY), _ptr(ws), ctypes.byref(g), _ptr(bws),
                              int(bws.numel()) * int(bws.element_size()),
                              _stream(stream)),
           "moe_backward")


def moe_backward_check(p, bws, stream=None) -> int:
    """Waits for the stream; MOE_ERR_TIMEOUT if a bounded wait of the last
    moe_backward on bws gave up, MOE_ERR_INVALID_ARG if its offsets_host
    differed from the forward's device offsets, else MOE_OK."""
    return lib().moe_backward_check(ctypes.byref(p), _ptr(bws), _stream(stream))
