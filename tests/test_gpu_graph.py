"""The forward pass enqueues no host synchronisation, allocation or device-to-host
copy, so it can be captured once into a CUDA graph and replayed (CUDA graphs take
the per-step CPU scheduling out of decode, Step3 推論最適化 (MI308X vs H20),
§最適化技術).  Replays must give the eager result bit for bit, on new inputs too."""
import pytest
import torch

import synth
from synth.workloads import Workload

from moe_harness import plan_for, to_device, weights_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    import mixture_experts_fp32_b200 as moe
    from mixture_experts_fp32_b200 import build
    build.build()
    moe.load()


@pytest.mark.parametrize("w", [
    Workload("graph_bf16", T=48, H=512, E=16, k=3, I=256, S=1, Is=256, router_sigma=0.2),
    Workload("graph_fp8", T=300, H=512, E=16, k=4, I=256, S=1, Is=128, wtype="fp8",
             router_sigma=0.2, w_sigma=0.05),
    Workload("graph_padded", T=1500, H=256, E=8, k=2, I=128, mask="dp_padded",
             dp_rows=(100, 3, 750)),
], ids=lambda w: w.name)
def test_graph_replay_matches_eager(w):
    inp = synth.make_inputs(w)
    d = to_device(inp)
    plan = plan_for(w)
    wts = weights_of(d)
    eager = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    plan.forward(wts, d["x"], d["valid"], w.k, eager)       # first call outside capture
    torch.cuda.synchronize()

    x_static = d["x"].clone()
    out_static = torch.empty_like(eager)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        plan.forward(wts, x_static, d["valid"], w.k, out_static)
    g.replay()
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    assert torch.equal(out_static.view(torch.int16), eager.view(torch.int16))

    # new hidden states in the captured buffer: replay follows them
    x2 = synth.normal_bf16(w.seed + 7, synth.STREAM_X, (w.T, w.H), 1.0).cuda()
    x_static.copy_(x2)
    g.replay()
    plan.forward(wts, x2, d["valid"], w.k, eager)
    torch.cuda.synchronize()
    assert torch.equal(out_static.view(torch.int16), eager.view(torch.int16))
    del g
