"""Forward passes of consecutive batches held in host memory, with the copies
overlapped.

Each batch is copied host -> device, runs moe_forward, and its output is
copied device -> host.  With two device buffers for x and Y and separate copy
streams, the upload of batch i+1 and the download of batch i-1 run while
batch i computes, so a stream of batches costs about max(compute, upload,
download) per batch instead of their sum.  Host buffers must be pinned.
torch provides the streams, events and copies; the layer itself runs in
libmoe's kernels.
"""
from __future__ import annotations

import sparse_mixture_experts_25_b200 as moe


class HostPipeline:
    def __init__(self, p: "moe.Params", weights: dict, depth: int = 2, x_dtype=None, device="cuda",
                 forward=None, ws_bytes=None, shape=None):
        """weights: device tensors W_r, W_g, W_u, W_d and optionally b_r, lat,
        Ws_g, Ws_u, Ws_d (held fixed across batches).  forward(x, y, ws,
        stream), if given, replaces moe_forward (for example the sharded
        forward of a multi-GPU routing group, or the Soft MoE forward, which
        passes p = None with its workspace bytes and the (N, d) shape)."""
        import torch
        self.torch = torch
        self.p = p
        self.w = weights
        self.forward = forward
        self.depth = depth
        N, d = shape if shape is not None else (p.N, p.d)
        bf16 = p is None or p.dtype == moe.MOE_BF16
        x_dtype = x_dtype or (torch.bfloat16 if bf16 else torch.float32)
        self.x = [torch.empty(N, d, dtype=x_dtype, device=device) for _ in range(depth)]
        self.y = [torch.empty(N, d, dtype=torch.float32, device=device) for _ in range(depth)]
        # batches compute one after another on one stream, so one workspace serves all
        nbytes = ws_bytes if ws_bytes is not None else moe.moe_workspace_size(p)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.compute = torch.cuda.Stream(device=device)
        self.h2d = torch.cuda.Stream(device=device)
        self.d2h = torch.cuda.Stream(device=device)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        self.uploaded = [ev() for _ in range(depth)]
        self.computed = [ev() for _ in range(depth)]
        self.downloaded = [ev() for _ in range(depth)]
        self.i = 0
        for b in range(depth):   # all buffers start free
            self.computed[b].record(self.compute)
            self.downloaded[b].record(self.d2h)

    def submit(self, x_host, y_host):
        """Queue one batch: x_host [N, d] pinned -> forward -> y_host [N, d]
        fp32 pinned.  Returns immediately; call synchronize() to wait."""
        torch, w, p = self.torch, self.w, self.p
        b = self.i % self.depth
        self.i += 1
        # x buffer b is free once the batch that last used it has computed
        self.h2d.wait_event(self.computed[b])
        with torch.cuda.stream(self.h2d):
            self.x[b].copy_(x_host, non_blocking=True)
            self.uploaded[b].record(self.h2d)
        # Y buffer b is free once its previous result has been downloaded
        self.compute.wait_event(self.uploaded[b])
        self.compute.wait_event(self.downloaded[b])
        with torch.cuda.stream(self.compute):
            if self.forward is not None:
                self.forward(self.x[b], self.y[b], self.ws, self.compute)
            else:
                moe.moe_forward(p, self.x[b], w["W_r"], w.get("b_r"), w.get("lat"), w["W_g"], w["W_u"],
                                w["W_d"], w.get("Ws_g"), w.get("Ws_u"), w.get("Ws_d"), self.y[b], self.ws,
                                self.compute)
            self.computed[b].record(self.compute)
        self.d2h.wait_event(self.computed[b])
        with torch.cuda.stream(self.d2h):
            y_host.copy_(self.y[b], non_blocking=True)
            self.downloaded[b].record(self.d2h)

    def synchronize(self):
        self.h2d.synchronize()
        self.compute.synchronize()
        self.d2h.synchronize()
