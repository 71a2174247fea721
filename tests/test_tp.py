"""Host side of the tensor-parallel layer: the shards reassemble the layer's weights, and
(the oracle, on the CPU) the sum of the shard layers' accumulators equals the whole
layer's, for bf16 and for FP8 block scales, so splitting the intermediate dimension is
exact and the slicing is right."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.workloads import Workload

from mixture_experts_fp32_b200 import tp

CASES = [
    Workload("tp_bf16", T=24, H=256, E=8, k=2, I=512, S=1, Is=512, router_sigma=0.2),
    Workload("tp_fp8", T=24, H=256, E=8, k=3, I=256, S=1, Is=256, wtype="fp8",
             router_sigma=0.2, w_sigma=0.05),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_shards_reassemble_the_layer(w):
    inp = synth.make_inputs(w)
    fp8 = w.wtype == "fp8"
    for n in (2, 4) if not fp8 else (2,):
        sh = [tp.shard_weights(inp, n, r, I=w.I, Is=w.Is, fp8=fp8) for r in range(n)]
        I, c = w.I, w.I // n
        gate = torch.cat([s["w_gate_up"][:, :c] for s in sh], dim=1)
        up = torch.cat([s["w_gate_up"][:, c:] for s in sh], dim=1)
        assert torch.equal(torch.cat([gate, up], dim=1), inp["w_gate_up"])
        assert torch.equal(torch.cat([s["w_down"] for s in sh], dim=2), inp["w_down"])
        cs = w.Is // n
        sgate = torch.cat([s["ws_gate_up"][:cs] for s in sh], dim=0)
        sup = torch.cat([s["ws_gate_up"][cs:] for s in sh], dim=0)
        assert torch.equal(torch.cat([sgate, sup]), inp["ws_gate_up"])
        assert torch.equal(torch.cat([s["ws_down"] for s in sh], dim=1), inp["ws_down"])
        if fp8:
            b = c // 128
            g = torch.cat([s["s_gate_up"][:, :b] for s in sh], dim=1)
            u = torch.cat([s["s_gate_up"][:, b:] for s in sh], dim=1)
            assert torch.equal(torch.cat([g, u], dim=1), inp["s_gate_up"])
            assert torch.equal(torch.cat([s["s_down"] for s in sh], dim=2), inp["s_down"])


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_shard_layers_sum_to_the_layer(w):
    inp = synth.make_inputs(w)
    fp8 = w.wtype == "fp8"
    full = oracle.forward(inp)
    for n in (2, 4) if not fp8 else (2,):
        acc = np.zeros_like(full["acc"])
        for r in range(n):
            sh = tp.shard_weights(inp, n, r, I=w.I, Is=w.Is, fp8=fp8)
            shard_inp = dict(inp)
            shard_inp.update(sh)
            shard_inp["workload"] = w.with_(I=w.I // n, Is=w.Is // n)
            acc += oracle.moe_tokens(shard_inp, full["ids"], full["w"])
        scale = np.abs(full["acc"]).max()
        assert np.abs(acc - full["acc"]).max() <= 1e-12 * scale


def test_a_wrong_slice_is_caught():
    # planted on the CPU side: swapping two shards' down columns breaks the identity
    w = CASES[0]
    inp = synth.make_inputs(w)
    full = oracle.forward(inp)
    shards = [tp.shard_weights(inp, 2, r, I=w.I, Is=w.Is, fp8=False) for r in range(2)]
    shards[0]["w_down"], shards[1]["w_down"] = shards[1]["w_down"], shards[0]["w_down"]
    acc = np.zeros_like(full["acc"])
    for sh in shards:
        shard_inp = dict(inp)
        shard_inp.update(sh)
        shard_inp["workload"] = w.with_(I=w.I // 2, Is=w.Is // 2)
        acc += oracle.moe_tokens(shard_inp, full["ids"], full["w"])
    assert np.abs(acc - full["acc"]).max() > 1e-3 * np.abs(full["acc"]).max()


def test_row_ownership_and_micro_batches():
    assert tp.owner_of(0, 1024) == (0, 0)
    assert tp.owner_of(4 * 1024 + 15, 1024) == (4, 15)
    assert tp.split_rows(1024) == ((0, 512), (512, 1024))
    assert tp.split_rows(7) == ((0, 3), (3, 7))


def test_shard_rejects_uneven_splits():
    w = CASES[1]
    inp = synth.make_inputs(w)
    with pytest.raises(ValueError):
        tp.shard_weights(inp, 3, 0, I=w.I, Is=w.Is, fp8=False)
    with pytest.raises(ValueError):
        tp.shard_weights(inp, 4, 0, I=w.I, Is=w.Is, fp8=True)   # 64-wide shard


@pytest.mark.parametrize("w", [
    Workload("ep_bf16", T=24, H=256, E=8, k=3, I=256, S=1, Is=512, router_sigma=0.2),
    Workload("ep_fp8", T=24, H=256, E=8, k=3, I=256, S=1, Is=256, wtype="fp8",
             router_sigma=0.2, w_sigma=0.05),
], ids=lambda w: w.name)
def test_expert_shards_sum_to_the_layer(w):
    """Expert-parallel layout: each rank's routed experts whole (pairs routed elsewhere
    contribute nothing there) plus 1/n of the shared expert; the ranks' accumulators,
    from the oracle on each rank's own weights, sum to the layer's."""
    inp = synth.make_inputs(w)
    fp8 = w.wtype == "fp8"
    full = oracle.forward(inp)
    ids, wts = full["ids"], full["w"]
    for n in (2, 4) if not fp8 else (2,):
        acc = np.zeros_like(full["acc"])
        for r in range(n):
            e0, e1 = tp.expert_range(w.E, n, r)
            sh = tp.shard_experts(inp, n, r, E=w.E, Is=w.Is, fp8=fp8)
            local = (ids >= e0) & (ids < e1)
            rank_inp = dict(inp)
            rank_inp.update(sh)
            rank_inp["workload"] = w.with_(E=e1 - e0, Is=w.Is // n)
            acc += oracle.moe_tokens(rank_inp, np.where(local, ids - e0, 0).astype(np.int32),
                                     np.where(local, wts, 0.0))
        assert np.abs(acc - full["acc"]).max() <= 1e-12 * np.abs(full["acc"]).max()
        assert tp.expert_range(w.E, n, n - 1)[1] == w.E
