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


@pytest.mark.parametrize("kw", [dict(fused=True), dict(fused=False),
                                dict(fused=True, layout="ep"),
                                dict(fused=True, layout="ep", pairs=True, send_ctas=8)],
                         ids=["tp-fused", "tp-nccl", "ep-fused", "ep-pairs"])
def test_one_rank_two_micro_batches(one_rank_group, kw):
    """Two micro-batches on one rank, in every return form (the per-pair one with its
    shared expert on the rank's own rows of each micro-batch): each micro-batch's
    rows equal the plain forward of that micro-batch, bit for bit, step after step."""
    w = Workload("tp1_tbo", T=96, H=512, E=16, k=3, I=512, S=1, Is=256, router_sigma=0.2,
                 mask="dp_padded", dp_rows=(70,))
    d = to_device(synth.make_inputs(w))
    refs = []
    for (lo, hi) in tp.split_rows(w.T):                  # each micro-batch is its own layer call
        sub = dict(d)
        sub["x"], sub["valid"] = d["x"][lo:hi], d["valid"][lo:hi]
        refs.append(run_forward(plan_for(w.with_(T=hi - lo)), sub, w.k)["out"])
    layer = tp.TPMoETwoBatch(d, E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is, k_max=w.k, rows=w.T,
                             fp8=False, **kw)
    for _ in range(3):                                   # alternate slabs across steps
        out = torch.full((w.T, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        layer.forward(d["x"], d["valid"], w.k, out)
        torch.cuda.synchronize()
        assert all(h.plan.device_status() == 0 for h in layer.halves)
        for (lo, hi), ref in zip(layer.ranges, refs):
            assert torch.equal(out[lo:hi].cpu().view(torch.int16), ref.view(torch.int16))


# ----------------------------------------------------- per-pair return (signalled sends)

PAIR_CASES = [
    (Workload("pairs1_bf16_padded", T=64, H=512, E=16, k=3, I=256, S=1, Is=256,
              router_sigma=0.2, mask="dp_padded", dp_rows=(40,)), 1),
    (Workload("pairs2_bf16_padded", T=4 * 48, H=512, E=16, k=3, I=256, S=1, Is=256,
              router_sigma=0.2, mask="dp_padded", dp_rows=(48, 5, 0, 17)), 2),
    (Workload("pairs4_bf16_zipf", T=4 * 64, H=512, E=16, k=4, I=256, S=1, Is=512,
              router_sigma=0.2, bias="zipf"), 4),
    (Workload("pairs2_fp8", T=2 * 64, H=512, E=8, k=2, I=256, S=1, Is=256, wtype="fp8",
              router_sigma=0.2, w_sigma=0.05), 2),
    (Workload("pairs4_fp8_no_shared", T=4 * 32, H=512, E=8, k=3, I=256, S=0, Is=0,
              wtype="fp8", router_sigma=0.2, w_sigma=0.05), 4),
    (Workload("pairs2_bf16_many_rows", T=2 * 400, H=256, E=4, k=2, I=256, S=1, Is=128,
              router_sigma=0.2), 2),                      # several row tiles per expert
]


@pytest.mark.parametrize("w,n", PAIR_CASES, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_emulated_pairs_return_matches_the_layer(w, n):
    """Each emulated expert-parallel rank computes the shared expert whole on its own
    rows and sends its routed experts' rows, one slot per pair, into the owners' slabs
    from the sender CTAs of its down GEMM; each owner's ordered sum is the one-GPU
    combine, so the owners' outputs equal the unsharded forward bit for bit (and the
    oracle within the layer's tolerance)."""
    inp = synth.make_inputs(w)
    d = to_device(inp)
    rows = w.T // n
    full_res = run_forward(plan_for(w), d, w.k)
    xs = [d["x"][r * rows:(r + 1) * rows] for r in range(n)]
    vs = [d["valid"][r * rows:(r + 1) * rows] for r in range(n)]
    for send_ctas in (1, 16):
        outs, statuses = tp.pairs_forward_reference(d, xs, vs, w.k, E=w.E, H=w.H, I=w.I, S=w.S,
                                                    Is=w.Is, fp8=w.wtype == "fp8", n_shards=n,
                                                    send_ctas=send_ctas)
        assert all(s == 0 for s in statuses), statuses
        got = torch.cat(outs).cpu()
        res = dict(full_res)
        res["out"] = got
        check_against_oracle(inp, res, w.k)
        assert torch.equal(got.view(torch.int16), full_res["out"].view(torch.int16))


def test_pairs_sender_wait_limit_sets_the_status_bit():
    """With a zero wait limit every wait not already satisfied gives up at once: the
    senders set MOE_DEV_WAIT_TIMEOUT_SEND and stop, the launch still ends, and the
    same plan then runs correctly with the normal limit."""
    w = Workload("pairs_timeout", T=2 * 64, H=512, E=8, k=2, I=256, S=0, Is=0,
                 router_sigma=0.2)
    inp = synth.make_inputs(w)
    d = to_device(inp)
    rows = w.T // 2
    shard = {"router_w": d["router_w"], "router_b": d.get("router_b"),
             "w_gate_up": d["w_gate_up"], "w_down": d["w_down"]}
    kern = tp.LibraryKernels(shard, E=w.E, H=w.H, inter=w.I, S=0, shared_inter=0, k_max=w.k,
                             T=w.T, fp8=False, device=d["x"].device)
    slabs = [torch.zeros(w.k + 1, rows, w.H, dtype=torch.float32, device="cuda")
             for _ in range(2)]
    kern.plan.set_wait_limit(0)
    kern.plan.forward_scatter_pairs(kern.weights, d["x"], d["valid"], w.k, slabs, rows, w.k,
                                    0, w.E, 8)
    torch.cuda.synchronize()
    bits = kern.plan.device_status()
    assert bits & moe.MOE_DEV_WAIT_TIMEOUT_SEND, hex(bits)
    kern.plan.set_wait_limit(2_000_000_000)
    wts = torch.empty(w.T, w.k, dtype=torch.float32, device="cuda")
    kern.plan.forward_scatter_pairs(kern.weights, d["x"], d["valid"], w.k, slabs, rows, w.k,
                                    0, w.E, 8, dbg=moe.make_debug(topk_w=wts))
    torch.cuda.synchronize()
    assert kern.plan.device_status() == 0
    ref = run_forward(plan_for(w), d, w.k)["out"]
    for r in range(2):
        o = torch.empty(rows, w.H, dtype=torch.bfloat16, device="cuda")
        moe.moe_reduce_pairs(slabs[r], w.k, 0, rows, w.H, wts[r * rows:(r + 1) * rows],
                             d["valid"][r * rows:(r + 1) * rows], o)
        torch.cuda.synchronize()
        assert torch.equal(o.cpu().view(torch.int16), ref[r * rows:(r + 1) * rows].view(torch.int16))


def test_one_rank_pairs_layer_equals_the_layer(one_rank_group):
    """TPMoE with the per-pair return on a one-rank group: the all_gather on the
    communication stream while the shared expert runs on the rank's own rows, the
    signalled sends into the symmetric-memory slab, the barrier and the owner's sum
    give the unsharded forward's output bit for bit, step after step."""
    w = Workload("pairs1_layer", T=64, H=512, E=16, k=3, I=512, S=1, Is=256, router_sigma=0.2,
                 mask="dp_padded", dp_rows=(40,))
    d = to_device(synth.make_inputs(w))
    ref = run_forward(plan_for(w), d, w.k)["out"]
    layer = tp.TPMoE(d, E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is, k_max=w.k, rows=w.T,
                     fp8=False, layout="ep", pairs=True, send_ctas=8)
    for _ in range(3):
        out = torch.full((w.T, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        layer.forward(d["x"], d["valid"], w.k, out)
        torch.cuda.synchronize()
        assert layer.plan.device_status() == 0
        assert torch.equal(out.cpu().view(torch.int16), ref.view(torch.int16))
