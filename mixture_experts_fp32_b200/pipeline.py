"""Host-to-host forwards whose copies overlap the compute of neighbouring batches.

A caller that keeps its hidden states in pinned host memory pays, for every batch,
an upload of x and the mask and a download of out.  Issued on the compute stream
they add to each step; here they run on their own copy streams, so the upload of
batch i+1 and the download of batch i-1 proceed on the copy engines while batch i
computes on the SMs.  Each of ``depth`` slots owns its device buffers (x, mask,
out); a slot is refilled only after its previous download has finished, and the
forwards share the plan's workspace by running one after another on the compute
stream.  With three slots the upload of batch i+1 need not wait for the download
of batch i-1, so a step costs the longest of the forward, the upload and the
download rather than the forward plus both copies.  With ``graph=True`` each
slot's forward is captured once as a CUDA graph over its static buffers and
replayed (the forward enqueues no host sync, allocation or device-to-host copy, so
it captures as is).
"""
from __future__ import annotations

import torch

from . import Plan, moe_weights


class HostPipeline:
    """Forwards of ``rows``-row batches from pinned host memory to pinned host memory.

    ``submit`` enqueues one batch and returns at once with an event that completes
    when the batch's output has reached ``out_host``; the caller keeps ``x_host`` and
    ``valid_host`` unchanged and ``out_host`` unread until then."""

    def __init__(self, plan: Plan, weights: moe_weights, k: int, rows: int, *, depth: int = 3,
                 graph: bool = True):
        if not 1 <= rows <= plan.cfg.max_tokens:
            raise ValueError(f"rows must be in [1, {plan.cfg.max_tokens}], got {rows}")
        if depth < 1:
            raise ValueError("depth must be at least 1")
        dev = plan.workspace.device
        H = plan.cfg.hidden
        self.plan, self.weights, self.k, self.rows, self.depth = plan, weights, k, rows, depth
        self.x = [torch.zeros(rows, H, dtype=torch.bfloat16, device=dev) for _ in range(depth)]
        self.valid = [torch.zeros(rows, dtype=torch.uint8, device=dev) for _ in range(depth)]
        self.out = [torch.empty(rows, H, dtype=torch.bfloat16, device=dev) for _ in range(depth)]
        self.up = torch.cuda.Stream(device=dev)
        self.compute = torch.cuda.Stream(device=dev)
        self.down = torch.cuda.Stream(device=dev)
        self.drained = [torch.cuda.Event() for _ in range(depth)]
        self.used = [False] * depth
        self.count = 0
        self.graphs = None
        # the first forward runs outside any capture (the library sets kernel
        # attributes on first use); all-padding batches, so it only writes zeros
        self.compute.wait_stream(torch.cuda.current_stream(dev))
        for s in range(depth):
            self._forward(s)
        if graph:
            self.compute.synchronize()
            self.graphs = []
            for s in range(depth):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=self.compute):
                    self._forward(s)
                self.graphs.append(g)
        self.compute.synchronize()

    def _forward(self, s: int) -> None:
        self.plan.forward(self.weights, self.x[s], self.valid[s], self.k, self.out[s],
                          stream=self.compute)

    def submit(self, x_host: torch.Tensor, valid_host, out_host: torch.Tensor) -> torch.cuda.Event:
        for name, t in (("x_host", x_host), ("valid_host", valid_host), ("out_host", out_host)):
            if t is not None and not t.is_pinned():
                raise ValueError(f"{name} must be in pinned host memory (so that copies overlap)")
        shape = tuple(self.x[0].shape)
        if tuple(x_host.shape) != shape or tuple(out_host.shape) != shape:
            raise ValueError(f"x_host and out_host must be [{self.rows}, {self.plan.cfg.hidden}]")
        if valid_host is not None and tuple(valid_host.shape) != (self.rows,):
            raise ValueError(f"valid_host must be [{self.rows}]")
        s = self.count % self.depth
        # refill a slot only after its previous output has been downloaded (which
        # itself followed that forward, the last reader of the slot's inputs)
        if self.used[s]:
            self.up.wait_event(self.drained[s])
        with torch.cuda.stream(self.up):
            self.x[s].copy_(x_host, non_blocking=True)
            if valid_host is None:
                self.valid[s].fill_(1)
            else:
                self.valid[s].copy_(valid_host, non_blocking=True)
        self.compute.wait_stream(self.up)
        with torch.cuda.stream(self.compute):
            if self.graphs is not None:
                self.graphs[s].replay()
            else:
                self._forward(s)
        self.down.wait_stream(self.compute)
        with torch.cuda.stream(self.down):
            out_host.copy_(self.out[s], non_blocking=True)
            self.drained[s].record(self.down)
            done = torch.cuda.Event()
            done.record(self.down)
        self.used[s] = True
        self.count += 1
        return done

    def synchronize(self) -> None:
        self.down.synchronize()

    def close(self) -> None:
        """Waits for the work in flight and releases the captured graphs."""
        self.synchronize()
        self.graphs = None
