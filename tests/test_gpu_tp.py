"""The tensor- and expert-parallel layers on one GPU.

* n shards emulated in one process: every shard's forward scatters its fp32 partial rows
  into every owner's slab, each owner sums its slab in rank order and rounds once; the
  owners' outputs must match the oracle's whole layer (same tolerance as the layer) and
  the unsharded forward, and padding rows must be +0.0.
* the same for the expert-parallel layout: each rank computes its own experts (pairs
  routed elsewhere left out of its permutation and combine) and 1/n of the shared expert;
* a one-rank NCCL process group runs the TPMoE class (fused path through symmetric
  memory, and the NCCL reduce_scatter path, both layouts) and the two-micro-batch
  schedule; with one rank the shard is the whole layer, so each must give the unsharded
  forward's output bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch

import synth
from synth.workloads import Workload

import mixture_experts_fp32_b200 as moe
from mixture_experts_fp32_b200 import tp

from moe_harness import check_against_oracle, plan_for, run_forward, to_device, weights_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_fp32_b200 import build
    build.build()
    moe.load()


CASES = [
    (Workload("tp2_bf16_padded", T=4 * 48, H=512, E=16, k=3, I=512, S=1, Is=256,
              router_sigma=0.2, mask="dp_padded", dp_rows=(48, 5, 0, 17)), 2, "tp"),
    (Workload("tp4_bf16_padded", T=4 * 48, H=512, E=16, k=3, I=512, S=1, Is=512,
              router_sigma=0.2, mask="dp_padded", dp_rows=(48, 5, 0, 17)), 4, "tp"),
    (Workload("tp2_fp8", T=2 * 64, H=512, E=8, k=2, I=256, S=1, Is=256, wtype="fp8",
              router_sigma=0.2, w_sigma=0.05), 2, "tp"),
    (Workload("ep2_bf16_padded", T=4 * 48, H=512, E=16, k=3, I=256, S=1, Is=256,
              router_sigma=0.2, mask="dp_padded", dp_rows=(48, 5, 0, 17)), 2, "ep"),
    (Workload("ep4_bf16_zipf", T=4 * 64, H=512, E=16, k=4, I=256, S=1, Is=512,
              router_sigma=0.2, bias="zipf"), 4, "ep"),
    (Workload("ep2_fp8", T=2 * 64, H=512, E=8, k=2, I=256, S=1, Is=256, wtype="fp8",
              router_sigma=0.2, w_sigma=0.05), 2, "ep"),
    (Workload("ep4_fp8_no_shared", T=4 * 32, H=512, E=8, k=3, I=256, S=0, Is=0, wtype="fp8",
              router_sigma=0.2, w_sigma=0.05), 4, "ep"),
]


@pytest.mark.parametrize("w,n,layout", CASES,
                         ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_emulated_ranks_match_the_layer(w, n, layout):
    inp = synth.make_inputs(w)
    d = to_device(inp)
    rows = w.T // n
    full_res = run_forward(plan_for(w), d, w.k)            # unsharded, with its logits
    xs = [d["x"][r * rows:(r + 1) * rows] for r in range(n)]
    vs = [d["valid"][r * rows:(r + 1) * rows] for r in range(n)]
    outs = tp.tp_forward_reference(d, xs, vs, w.k, E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is,
                                   k_max=w.k, fp8=w.wtype == "fp8", n_shards=n, layout=layout)
    got = torch.cat(outs).cpu()
    res = dict(full_res)
    res["out"] = got
    rep = check_against_oracle(inp, res, w.k)                # tolerance, routing, +0.0 padding
    diff = (got.float() - full_res["out"].float()).abs()
    scale = full_res["out"].float().abs().max()
    assert float(diff.max()) <= 2 ** -7 * float(scale), rep   # same sums, other fp32 order


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.fixture(scope="module")
def one_rank_group():
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), RANK="0",
                      WORLD_SIZE="1")
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0),
                            timeout=__import__("datetime").timedelta(seconds=60))
    yield None
    dist.destroy_process_group()


@pytest.mark.parametrize("fused,layout", [(True, "tp"), (False, "tp"), (True, "ep")],
                         ids=["tp-fused", "tp-nccl", "ep-fused"])
def test_one_rank_tp_equals_the_layer(one_rank_group, fused, layout):
    w = Workload("tp1", T=64, H=512, E=16, k=3, I=512, S=1, Is=256, router_sigma=0.2,
                 mask="dp_padded", dp_rows=(40,))
    d = to_device(synth.make_inputs(w))
    ref = run_forward(plan_for(w), d, w.k)["out"]
    layer = tp.TPMoE(d, E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is, k_max=w.k, rows=w.T,
                     fp8=False, fused=fused, layout=layout)
    for _ in range(3):                                   # alternate slabs across steps
        out = torch.full((w.T, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        layer.forward(d["x"], d["valid"], w.k, out)
        torch.cuda.synchronize()
        assert layer.plan.device_status() == 0
        assert torch.equal(out.cpu().view(torch.int16), ref.view(torch.int16))


def test_one_rank_two_micro_batches(one_rank_group):
    w = Workload("tp1_tbo", T=96, H=512, E=16, k=3, I=512, S=1, Is=256, router_sigma=0.2,
                 mask="dp_padded", dp_rows=(70,))
    d = to_device(synth.make_inputs(w))
    layer = tp.TPMoETwoBatch(d, E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is, k_max=w.k, rows=w.T,
                             fp8=False, fused=True)
    out = torch.full((w.T, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    layer.forward(d["x"], d["valid"], w.k, out)
    torch.cuda.synchronize()
    for (lo, hi) in layer.ranges:                        # each micro-batch is its own layer call
        sub = dict(d)
        sub["x"], sub["valid"] = d["x"][lo:hi], d["valid"][lo:hi]
        sub["workload"] = w.with_(T=hi - lo)
        ref = run_forward(plan_for(sub["workload"]), sub, w.k)["out"]
        assert torch.equal(out[lo:hi].cpu().view(torch.int16), ref.view(torch.int16))
