"""The tensor- and expert-parallel layers' host side on two and four gloo ranks (CPU).

TPMoE's own steps run for real: the all_gather of every rank's rows and masks, the
collective return (reduce_scatter of the fp32 partials), the row ownership and each
owner's slice of the result.  Its two compute steps, which the library runs on the GPU,
are stood in for by the oracle: a rank's forward is the oracle's accumulator of its
shard layer over the gathered rows (routing over all experts; pairs of other ranks'
experts weighted 0 in the expert-parallel layout), stored as fp32 rows; the owner's
step sums the slots in order and rounds once to bf16, padding rows +0.0.  The owners'
outputs must then equal the oracle's whole layer up to that fp32 rounding.

Failure: a rank that fails before the step leaves the other one's all_gather to end
with an error (the process group's timeout) rather than wait."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

WORKLOADS = {
    "tp_padded": dict(T=2 * 24, H=256, E=8, k=2, I=256, S=1, Is=256, router_sigma=0.2,
                      mask="dp_padded", dp_rows=(24, 7)),
    "ep_zipf": dict(T=2 * 24, H=256, E=8, k=3, I=128, S=1, Is=256, router_sigma=0.2,
                    bias="zipf"),
    "ep_fp8_no_shared": dict(T=2 * 16, H=256, E=4, k=2, I=128, S=0, Is=0, wtype="fp8",
                             router_sigma=0.2, w_sigma=0.05),
    "tp_fp8": dict(T=2 * 16, H=256, E=8, k=2, I=256, S=1, Is=256, wtype="fp8",
                   router_sigma=0.2, w_sigma=0.05),
    "tp4_padded": dict(T=4 * 16, H=256, E=8, k=3, I=512, S=1, Is=512, router_sigma=0.2,
                       mask="dp_padded", dp_rows=(16, 3, 0, 9)),
    "ep4": dict(T=4 * 16, H=256, E=8, k=2, I=128, S=1, Is=512, router_sigma=0.2),
}
LAYOUT = {"tp_padded": "tp", "ep_zipf": "ep", "ep_fp8_no_shared": "ep", "tp_fp8": "tp",
          "tp4_padded": "tp", "ep4": "ep"}
WORLD = {"tp4_padded": 4, "ep4": 4}


class OracleKernels:
    """The two compute steps of a rank, computed by the oracle on the CPU."""

    def __init__(self, shard, *, E, H, inter, S, shared_inter, k_max, T, fp8, device):
        self.shard, self.E, self.H = shard, E, H
        self.inter, self.S, self.Is, self.fp8 = inter, S, shared_inter, fp8
        self.plan = None

    def forward_scatter_experts(self, x_all, valid_all, k, dst, rows_per_rank, slot, e0, e1):
        import oracle
        from synth.workloads import Workload
        T = x_all.shape[0]
        logits = oracle.router_logits(x_all, valid_all, self.shard["router_w"],
                                      self.shard.get("router_b"))
        ids, w = oracle.topk(logits, valid_all, k)
        local = (ids >= e0) & (ids < e1)
        inputs = dict(self.shard)
        inputs["x"] = x_all
        inputs["workload"] = Workload("rank", T=T, H=self.H, E=e1 - e0, k=k, I=self.inter,
                                      S=self.S, Is=self.Is, wtype="fp8" if self.fp8 else "bf16")
        acc = oracle.moe_tokens(inputs, np.where(local, ids - e0, 0).astype(np.int32),
                                np.where(local, w, 0.0))
        acc[valid_all.numpy() == 0] = 0.0
        part = torch.from_numpy(acc.astype(np.float32))
        for t in range(T):
            owner, lt = divmod(t, rows_per_rank)
            dst[owner].view(-1, self.H)[slot * rows_per_rank + lt] = part[t]

    def reduce_partials(self, slab, n_slots, rows, H, valid, out):
        s = slab.view(n_slots, rows, H)
        acc = s[0].clone()
        for g in range(1, n_slots):
            acc += s[g]
        o = acc.to(torch.bfloat16)
        o[valid == 0] = 0.0
        out.copy_(o)


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank: int, world: int, port: int, name: str, q):
    import torch.distributed as dist
    import synth
    from synth.workloads import Workload
    from mixture_experts_fp32_b200 import tp
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = Workload(name, **WORKLOADS[name])
        inp = synth.make_inputs(w)
        rows = w.T // world
        layer = tp.TPMoE(inp, E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is, k_max=w.k, rows=rows,
                         fp8=w.wtype == "fp8", fused=False, layout=LAYOUT[name],
                         kernels=OracleKernels)
        x_local = inp["x"][rank * rows:(rank + 1) * rows].contiguous()
        v_local = inp["valid"][rank * rows:(rank + 1) * rows].contiguous()
        out = torch.full((rows, w.H), float("nan"), dtype=torch.bfloat16)
        layer.forward(x_local, v_local, w.k, out)
        q.put((rank, out.view(torch.int16).numpy().copy()))
    finally:
        dist.destroy_process_group()


def _spawn(target, args_of, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, *args_of(r), q))
             for r in range(world)]
    for p in procs:
        p.start()
    return procs, q


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_ranks_return_the_layer(name):
    import oracle
    import synth
    from synth.workloads import Workload
    world = WORLD.get(name, 2)
    procs, q = _spawn(_rank_main, lambda r: (name,), world=world)
    got = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    w = Workload(name, **WORKLOADS[name])
    inp = synth.make_inputs(w)
    ref = oracle.forward(inp)
    out = np.concatenate([got[r] for r in range(world)]).view(np.uint16)
    ref_f = oracle.bf16_to_f64(ref["out"])
    out_f = oracle.bf16_to_f64(out)
    valid = inp["valid"].numpy().astype(bool)
    scale = np.abs(ref["acc"][valid]).max()
    # per-rank fp32 partials, one fp32 sum, one rounding: within a bf16 step of the layer
    assert np.abs(out_f - ref_f)[valid].max() <= 2.0 ** -7 * scale
    assert (out[~valid] == 0).all()                    # padding rows +0.0


def _failing_rank_main(rank: int, world: int, port: int, q):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(3)                                    # dies before the step
    from mixture_experts_fp32_b200 import tp
    import synth
    from synth.workloads import Workload
    w = Workload("tp_padded", **WORKLOADS["tp_padded"])
    inp = synth.make_inputs(w)
    rows = w.T // world
    try:
        layer = tp.TPMoE(inp, E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is, k_max=w.k, rows=rows,
                         fused=False, kernels=OracleKernels)
        layer.forward(inp["x"][:rows].contiguous(), inp["valid"][:rows].contiguous(), w.k,
                      torch.empty(rows, w.H, dtype=torch.bfloat16))
        q.put((rank, "completed"))
    except Exception as e:                             # the collective gave up
        q.put((rank, type(e).__name__))


def test_a_failed_rank_ends_the_others_collective_with_an_error():
    procs, q = _spawn(_failing_rank_main, lambda r: ())
    rank, what = q.get(timeout=120)
    for p in procs:
        p.join(60)
    assert rank == 0 and what != "completed"
    assert procs[1].exitcode == 3
