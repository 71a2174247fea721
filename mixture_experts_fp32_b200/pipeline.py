"""Host-to-host forwards whose copies overlap the compute of neighbouring batches.

A thin wrapper over the library's pipeline (``moe_pipeline_*`` in the C ABI): the
library uploads each batch's hidden states and mask from host memory and downloads
its output on two copy streams of its own, beside a compute stream that runs the
forwards, so the upload of batch i+1 and the download of batch i-1 proceed on the
copy engines while batch i computes.  Each of ``depth`` slots owns device buffers
for one batch (allocated here, by torch, and handed to the library); a slot is
refilled only after its previous download has finished.  With three slots a step
costs the longest of the forward, the upload and the download rather than their
sum.  With ``graph=True`` each slot's forward is captured once as a CUDA graph and
replayed.
"""
from __future__ import annotations

import torch

from . import (Plan, moe_pipeline_create, moe_pipeline_destroy, moe_pipeline_slot_bytes,
               moe_pipeline_streams, moe_pipeline_submit, moe_pipeline_synchronize, moe_weights)


class HostPipeline:
    """Forwards of ``rows``-row batches from page-locked host memory to page-locked
    host memory.  ``submit`` enqueues one batch and returns; the caller keeps
    ``x_host`` and ``valid_host`` unchanged and ``out_host`` unread until
    ``synchronize()`` (or an event recorded on ``self.down`` after the submit) says
    the batch is done.  Creating it synchronises the device."""

    def __init__(self, plan: Plan, weights: moe_weights, k: int, rows: int, *, depth: int = 3,
                 graph: bool = True):
        self.plan, self.rows, self.depth = plan, rows, depth
        dev = plan.workspace.device
        nbytes = moe_pipeline_slot_bytes(plan.handle, rows, depth)
        self.slots = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.handle = moe_pipeline_create(plan.handle, weights, k, rows, depth, graph, self.slots,
                                          nbytes, plan.workspace, plan.ws_bytes)
        up, compute, down = moe_pipeline_streams(self.handle)
        self.up = torch.cuda.ExternalStream(up, device=dev)
        self.compute = torch.cuda.ExternalStream(compute, device=dev)
        self.down = torch.cuda.ExternalStream(down, device=dev)

    def submit(self, x_host: torch.Tensor, valid_host, out_host: torch.Tensor) -> None:
        for name, t in (("x_host", x_host), ("valid_host", valid_host), ("out_host", out_host)):
            if t is not None and not t.is_pinned():
                raise ValueError(f"{name} must be in pinned host memory (so that copies overlap)")
        shape = (self.rows, self.plan.cfg.hidden)
        if tuple(x_host.shape) != shape or tuple(out_host.shape) != shape:
            raise ValueError(f"x_host and out_host must be [{shape[0]}, {shape[1]}]")
        if valid_host is not None and tuple(valid_host.shape) != (self.rows,):
            raise ValueError(f"valid_host must be [{self.rows}]")
        moe_pipeline_submit(self.handle, x_host, valid_host, out_host)

    def synchronize(self) -> None:
        moe_pipeline_synchronize(self.handle)

    def close(self) -> None:
        """Waits for the batches in flight and releases the library's pipeline."""
        if self.handle:
            moe_pipeline_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
