"""Host-to-host forwards through the library's pipeline (moe_pipeline_*, wrapped by
HostPipeline: copies on their own streams, slots reused, optionally graph-replayed)
give, batch for batch, the bits of the plain forward on the same inputs."""
import pytest
import torch

import synth
from synth.workloads import Workload

import mixture_experts_fp32_b200 as moe
from mixture_experts_fp32_b200.pipeline import HostPipeline

from moe_harness import plan_for, to_device, weights_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_fp32_b200 import build
    build.build()
    moe.load()


W = Workload("pipe", T=96, H=512, E=16, k=3, I=256, S=1, Is=256, router_sigma=0.2)


def _batches(n, rows, H):
    g = torch.Generator().manual_seed(5)
    xs, vs = [], []
    for i in range(n):
        xs.append(torch.randn(rows, H, generator=g).to(torch.bfloat16).pin_memory())
        v = (torch.rand(rows, generator=g) > 0.25).to(torch.uint8)
        if i == 2:
            v.zero_()                                  # an all-padding batch in the stream
        vs.append(v.pin_memory())
    return xs, vs


@pytest.mark.parametrize("graph,depth", [(True, 3), (False, 2), (True, 1)])
def test_pipeline_matches_plain_forward(graph, depth):
    d = to_device(synth.make_inputs(W))
    plan = plan_for(W)
    wts = weights_of(d)
    xs, vs = _batches(7, W.T, W.H)
    refs = []
    for x, v in zip(xs, vs):
        out = torch.empty(W.T, W.H, dtype=torch.bfloat16, device="cuda")
        plan.forward(wts, x.cuda(), v.cuda(), W.k, out)
        refs.append(out.cpu())
    pipe = HostPipeline(plan, wts, W.k, W.T, depth=depth, graph=graph)
    outs = [torch.full((W.T, W.H), float("nan"), dtype=torch.bfloat16).pin_memory()
            for _ in xs]
    for x, v, o in zip(xs, vs, outs):
        pipe.submit(x, v, o)
    pipe.synchronize()
    pipe.close()
    assert plan.device_status() == 0
    for i, (o, r) in enumerate(zip(outs, refs)):
        assert torch.equal(o.view(torch.int16), r.view(torch.int16)), i
    assert (outs[2].view(torch.int16) == 0).all()      # all padding: +0.0 everywhere


def test_pipeline_refuses_pageable_or_misshaped_buffers():
    d = to_device(synth.make_inputs(W))
    plan = plan_for(W)
    pipe = HostPipeline(plan, weights_of(d), W.k, W.T, graph=False)
    x = torch.zeros(W.T, W.H, dtype=torch.bfloat16)
    out = torch.zeros(W.T, W.H, dtype=torch.bfloat16).pin_memory()
    with pytest.raises(ValueError, match="pinned"):
        pipe.submit(x, None, out)
    with pytest.raises(ValueError, match="x_host"):
        pipe.submit(x[:-1].pin_memory(), None, out)
    pipe.close()
