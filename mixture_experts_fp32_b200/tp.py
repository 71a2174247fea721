"""Tensor-parallel MoE behind data-parallel attention ranks.

DP attention in front of a TP MoE, joined by standard collectives (DP Attention and
TBO for DeepSeek-V4 on MI355X, introduction): every rank all_gathers the hidden rows of
all DP ranks, computes the whole layer for them with its 1/n share of every expert's
intermediate dimension, and the n partial outputs are summed back to the rank that owns
each row.  Splitting the intermediate dimension is exact: with gate/up rows and down
columns split alike, sum over shards of the shard layers equals the layer (the 1x128
activation groups of the FP8 path stay whole when I/n is a multiple of 128).  Routing is
computed by every rank from the same gathered rows and the same router, so all ranks
agree without exchanging it.

Two ways to return the partial sums:
  * fused: the library's combine writes each row's fp32 partial straight into the
    owner's receive slab (symmetric memory, peer pointers; `moe_forward_scatter`), a
    device barrier (bounded) tells every owner that all contributions have landed, and
    the owner sums its slab in rank order and rounds once (`moe_reduce_partials`);
  * nccl: the fp32 partial [n * rows, H] goes through NCCL's reduce_scatter, then is
    rounded by `moe_reduce_partials` with one slot.
The fused form needs no copy of the partial and sums in the same order on every owner.

Two micro-batches (TBO at the collective boundaries, same page, §最大の見どころ): the
local rows are split in two; the all_gather of the second runs on a communication stream
while the first computes, and (nccl form) the first's reduce_scatter runs while the
second computes.

Expert parallelism uses the same gather and the same return: rank r owns the routed
experts [r E/n, (r+1) E/n) (and 1/n of the shared expert's intermediate dimension);
routing is still computed over all experts, pairs routed elsewhere are left out of its
permutation (`moe_forward_scatter_experts`), and its combine returns each token's sum
over its own experts.  The all_gather stands in for the dispatch and the fused partial
return for the combine's all-to-all, so no kernel waits on another (the down GEMM's
per-expert completion signals of an all-to-all combine are not needed: the return rides
in the layer's last kernel).

Per-pair return ("pairs", expert-parallel layout; the Single Batch Overlap of the
[SGLang] MoE 모델을 위한 Single Batch Overlap 기법 page): the shared expert is computed
whole by every rank on its own rows, while its all_gather (the dispatch) is in flight;
the routed experts' down GEMM raises a completion counter per expert, and sender CTAs
of the same launch copy each finished expert's output rows, unweighted, into slot j of
the owning rank's slab as soon as that expert is done (`moe_forward_scatter_pairs`);
the owner then sums its k slots with its routing weights in the one-GPU order, plus
the shared row (`moe_reduce_pairs`).

Row ownership: gathered row t belongs to rank t // rows, local row t % rows.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import torch

import mixture_experts_fp32_b200 as moe


def shard_weights(full: Dict[str, Optional[torch.Tensor]], n: int, r: int, *, I: int, Is: int,
                  fp8: bool) -> Dict[str, Optional[torch.Tensor]]:
    """Rank r's share (1/n of every expert's intermediate dimension) of the layer's
    weights, as contiguous tensors on the same device.

    w_gate_up [E, 2I, H]: gate rows [r I/n, (r+1) I/n) and the same up rows (offset I);
    w_down [E, H, I]: the same columns; FP8 block scales [E, 2I/128, H/128] and
    [E, H/128, I/128] follow their 128-blocks; the shared expert likewise with Is."""
    if I % (128 * n) or (Is and Is % (128 * n)):
        raise ValueError("each rank's share of the intermediate dimensions must be a multiple "
                         "of 128 (the GEMM tiles and the FP8 blocks)")
    i0, i1 = r * I // n, (r + 1) * I // n
    out = {"router_w": full["router_w"], "router_b": full.get("router_b")}
    wgu = full["w_gate_up"]
    out["w_gate_up"] = torch.cat([wgu[:, i0:i1], wgu[:, I + i0:I + i1]], dim=1).contiguous()
    out["w_down"] = full["w_down"][:, :, i0:i1].contiguous()
    if fp8:
        b0, b1, bI = i0 // 128, i1 // 128, I // 128
        sgu = full["s_gate_up"]
        out["s_gate_up"] = torch.cat([sgu[:, b0:b1], sgu[:, bI + b0:bI + b1]], dim=1).contiguous()
        out["s_down"] = full["s_down"][:, :, b0:b1].contiguous()
    out.update(_shard_shared(full, n, r, Is=Is, fp8=fp8))
    return out


def _shard_shared(full, n: int, r: int, *, Is: int, fp8: bool) -> dict:
    """1/n of the shared expert's intermediate dimension (empty dict without one)."""
    out = {}
    if full.get("ws_gate_up") is None:
        return out
    if Is % (128 * n):
        raise ValueError("each rank's share of the shared expert must be a multiple of 128")
    j0, j1 = r * Is // n, (r + 1) * Is // n
    ws = full["ws_gate_up"]
    out["ws_gate_up"] = torch.cat([ws[j0:j1], ws[Is + j0:Is + j1]], dim=0).contiguous()
    out["ws_down"] = full["ws_down"][:, j0:j1].contiguous()
    if fp8:
        c0, c1, cI = j0 // 128, j1 // 128, Is // 128
        ss = full["ss_gate_up"]
        out["ss_gate_up"] = torch.cat([ss[c0:c1], ss[cI + c0:cI + c1]], dim=0).contiguous()
        out["ss_down"] = full["ss_down"][:, c0:c1].contiguous()
    return out


def expert_range(E: int, n: int, r: int):
    """The routed experts rank r owns in the expert-parallel layout."""
    if E % n:
        raise ValueError("the routed experts must divide by the number of ranks")
    return r * E // n, (r + 1) * E // n


def shard_experts(full: Dict[str, Optional[torch.Tensor]], n: int, r: int, *, E: int, Is: int,
                  fp8: bool) -> Dict[str, Optional[torch.Tensor]]:
    """Rank r's share in the expert-parallel layout: its routed experts whole, and 1/n
    of the shared expert's intermediate dimension (as in the tensor-parallel shard)."""
    e0, e1 = expert_range(E, n, r)
    out = {"router_w": full["router_w"], "router_b": full.get("router_b")}
    out["w_gate_up"] = full["w_gate_up"][e0:e1].contiguous()
    out["w_down"] = full["w_down"][e0:e1].contiguous()
    if fp8:
        out["s_gate_up"] = full["s_gate_up"][e0:e1].contiguous()
        out["s_down"] = full["s_down"][e0:e1].contiguous()
    out.update(_shard_shared(full, n, r, Is=Is, fp8=fp8))
    return out


def make_shard_weights(sh: Dict[str, Optional[torch.Tensor]],
                       router_split=None) -> moe.moe_weights:
    return moe.make_weights(sh["router_w"], sh.get("router_b"), sh["w_gate_up"], sh["w_down"],
                            sh.get("s_gate_up"), sh.get("s_down"), sh.get("ws_gate_up"),
                            sh.get("ws_down"), sh.get("ss_gate_up"), sh.get("ss_down"),
                            router_split)


def owner_of(t: int, rows: int):
    """(owning rank, local row) of gathered row t."""
    return t // rows, t % rows


def split_rows(rows: int):
    """The two micro-batches of a rank's rows: [0, a) and [a, rows), a = rows // 2."""
    a = rows // 2
    return (0, a), (a, rows)


class LibraryKernels:
    """A rank's compute steps, run by the library on the GPU: the forward over the
    gathered rows that stores each token's fp32 partial into the owners' slabs
    (`moe_forward_scatter_experts`), and the owner's ordered sum and rounding
    (`moe_reduce_partials`)."""

    def __init__(self, shard: dict, *, E: int, H: int, inter: int, S: int, shared_inter: int,
                 k_max: int, T: int, fp8: bool, device):
        self.plan = moe.Plan(max_tokens=T, hidden=H, num_experts=E, top_k_max=k_max,
                             inter=inter, num_shared=S, shared_inter=shared_inter,
                             wtype=moe.MOE_W_FP8_E4M3_B128 if fp8 else moe.MOE_W_BF16,
                             device=device)
        # the router weights' bf16 split, made once here rather than in every forward
        nbytes = moe.moe_router_split_bytes(self.plan.handle)
        self.router_split = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=device)
        moe.moe_split_router_weights(self.plan.handle, shard["router_w"], self.router_split,
                                     nbytes)
        self.weights = make_shard_weights(shard, router_split=self.router_split)

    def forward_scatter_experts(self, x_all, valid_all, k, dst, rows_per_rank, slot, e0, e1):
        self.plan.forward_scatter_experts(self.weights, x_all, valid_all, k, dst, rows_per_rank,
                                          slot, e0, e1)

    def reduce_partials(self, slab, n_slots, rows, H, valid, out):
        moe.moe_reduce_partials(slab, n_slots, rows, H, valid, out)


class SharedOwnRows:
    """The shared expert of the per-pair layout, whole, on a rank's own rows: a
    one-expert layer whose router always picks that expert with weight exactly 1
    (zero router weights), returned unrounded into the rank's own slab."""

    def __init__(self, full: dict, *, H: int, Is: int, rows: int, fp8: bool, device):
        self.plan = moe.Plan(max_tokens=rows, hidden=H, num_experts=1, top_k_max=1, inter=Is,
                             wtype=moe.MOE_W_FP8_E4M3_B128 if fp8 else moe.MOE_W_BF16,
                             device=device)
        self.router_w = torch.zeros(1, H, dtype=torch.float32, device=device)
        self.w_gate_up = full["ws_gate_up"][None].contiguous()
        self.w_down = full["ws_down"][None].contiguous()
        self.s_gate_up = full["ss_gate_up"][None].contiguous() if fp8 else None
        self.s_down = full["ss_down"][None].contiguous() if fp8 else None
        self.weights = self.plan.weights(self.router_w, None, self.w_gate_up, self.w_down,
                                         self.s_gate_up, self.s_down)

    def forward(self, x_local, valid_local, dst_ptr: int, rows: int, stream=None):
        self.plan.forward_scatter(self.weights, x_local, valid_local, 1, [dst_ptr], rows, 0,
                                  stream=stream)


class TPMoE:
    """One rank of the tensor-parallel layer (layout "tp") or of the expert-parallel one
    (layout "ep").  `full` holds the whole layer's weights on this rank's device (the
    shard is cut from it); `rows` is the number of rows each DP rank contributes per
    micro-batch (padding rows included, marked invalid).

    ``kernels`` builds the compute steps from (shard, E, H, inter, S, shared_inter, k_max,
    T, fp8, device); the default is the library (:class:`LibraryKernels`).  The
    collectives, the row ownership and the slab layout are this class's own, so that a
    stand-in for the two compute steps can run them on CPU ranks (the collective return
    only: the fused one needs peer-mapped device memory)."""

    def __init__(self, full: dict, *, E: int, H: int, I: int, S: int, Is: int, k_max: int,
                 rows: int, fp8: bool = False, fused: bool = True, group=None,
                 barrier_timeout_ms: int = 10000, layout: str = "tp", kernels=LibraryKernels,
                 pairs: bool = False, send_ctas: int = 16):
        import torch.distributed as dist
        self.group = group if group is not None else dist.group.WORLD
        self.n = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if self.n > moe.MAX_TP_RANKS:
            raise ValueError("at most 8 tensor-parallel ranks")
        self.H, self.rows, self.fused = H, rows, fused
        self.timeout_ms = barrier_timeout_ms
        self.pairs = pairs
        if pairs:
            self._init_pairs(full, E=E, H=H, I=I, S=S, Is=Is, k_max=k_max, rows=rows, fp8=fp8,
                             send_ctas=send_ctas)
            return
        if layout == "tp":
            self.shard = shard_weights(full, self.n, self.rank, I=I, Is=Is, fp8=fp8)
            self.experts, inter = (0, E), I // self.n
        elif layout == "ep":
            self.shard = shard_experts(full, self.n, self.rank, E=E, Is=Is, fp8=fp8)
            self.experts, inter = expert_range(E, self.n, self.rank), I
        else:
            raise ValueError(layout)
        dev = full["w_gate_up"].device
        T = self.n * rows
        self.kernels = kernels(self.shard, E=E, H=H, inter=inter, S=S,
                               shared_inter=Is // self.n if S else 0, k_max=k_max, T=T,
                               fp8=fp8, device=dev)
        self.x_all = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.valid_all = torch.empty(T, dtype=torch.uint8, device=dev)
        self.step = 0
        if fused:
            import torch.distributed._symmetric_memory as symm
            # two slabs, used on alternate steps: a rank may write step s+1's rows into
            # an owner's slab only after that owner has reduced step s-1 from it, which
            # the barrier of step s guarantees (each rank reduces s-1 before it scatters s)
            self.slab = symm.empty(2, self.n, rows, H, dtype=torch.float32, device=dev)
            self.handle = symm.rendezvous(self.slab, self.group)
            base = [int(p) for p in self.handle.buffer_ptrs]
            per = self.n * rows * H * 4
            self.dst = [[b + par * per for b in base] for par in range(2)]
        else:
            self.partial = torch.empty(T, H, dtype=torch.float32, device=dev)
            self.recv = torch.empty(rows, H, dtype=torch.float32, device=dev)

    def _init_pairs(self, full, *, E, H, I, S, Is, k_max, rows, fp8, send_ctas):
        """Expert-parallel layout with the per-pair return: this rank's routed experts
        whole (no shared expert in that plan), the shared expert whole on its own rows,
        and a slab of k_max + 1 slots per owner (two, used on alternate steps)."""
        import torch.distributed._symmetric_memory as symm
        dev = full["w_gate_up"].device
        self.experts = expert_range(E, self.n, self.rank)
        e0, e1 = self.experts
        self.shard = {"router_w": full["router_w"], "router_b": full.get("router_b"),
                      "w_gate_up": full["w_gate_up"][e0:e1].contiguous(),
                      "w_down": full["w_down"][e0:e1].contiguous()}
        if fp8:
            self.shard["s_gate_up"] = full["s_gate_up"][e0:e1].contiguous()
            self.shard["s_down"] = full["s_down"][e0:e1].contiguous()
        T = self.n * rows
        self.kernels = LibraryKernels(self.shard, E=E, H=H, inter=I, S=0, shared_inter=0,
                                      k_max=k_max, T=T, fp8=fp8, device=dev)
        self.shared = (SharedOwnRows(full, H=H, Is=Is, rows=rows, fp8=fp8, device=dev)
                       if S else None)
        self.k_max, self.send_ctas = k_max, send_ctas
        self.x_all = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.valid_all = torch.empty(T, dtype=torch.uint8, device=dev)
        self.w_all = torch.empty(T, k_max, dtype=torch.float32, device=dev)
        self.step = 0
        self.slab = symm.empty(2, k_max + 1, rows, H, dtype=torch.float32, device=dev)
        self.handle = symm.rendezvous(self.slab, self.group)
        base = [int(p) for p in self.handle.buffer_ptrs]
        per = (k_max + 1) * rows * H * 4
        self.dst = [[b + par * per for b in base] for par in range(2)]
        self.comm = torch.cuda.Stream(device=dev)

    def _forward_pairs(self, x_local, valid_local, k: int, out_local):
        main = torch.cuda.current_stream()
        # the dispatch (all_gather) on the communication stream, while the shared
        # expert runs on this rank's own rows
        self.comm.wait_stream(main)
        with torch.cuda.stream(self.comm):
            self._gather(x_local, valid_local)
        self._shared_own(x_local, valid_local)
        main.wait_stream(self.comm)
        self._compute_and_return(k, valid_local, out_local)

    def _shared_own(self, x_local, valid_local):
        """Per-pair layout: the shared expert on this rank's own rows, into its own
        slab's last slot (nothing without a shared expert or in the other layouts)."""
        if self.pairs and self.shared is not None:
            own = self.dst[self.step & 1][self.rank] + self.k_max * self.rows * self.H * 4
            self.shared.forward(x_local, valid_local, own, self.rows)

    def _return_pairs(self, k: int, valid_local, out_local):
        if k != self.k_max:
            raise ValueError("the per-pair slabs and weights are laid out for k = k_max")
        par = self.step & 1
        dbg = moe.make_debug(topk_w=self.w_all)
        self.kernels.plan.forward_scatter_pairs(self.kernels.weights, self.x_all, self.valid_all,
                                                k, self.dst[par], self.rows, k, *self.experts,
                                                self.send_ctas, dbg=dbg)
        self.handle.barrier(channel=0, timeout_ms=self.timeout_ms)
        lo = self.rank * self.rows
        moe.moe_reduce_pairs(self.slab[par], k, 1 if self.shared is not None else 0, self.rows,
                             self.H, self.w_all[lo:lo + self.rows], valid_local, out_local)

    @property
    def plan(self):
        return self.kernels.plan

    def _gather(self, x_local, valid_local):
        import torch.distributed as dist
        dist.all_gather_into_tensor(self.x_all, x_local, group=self.group)
        dist.all_gather_into_tensor(self.valid_all, valid_local, group=self.group)

    def _compute_and_return(self, k: int, valid_local, out_local):
        """The layer over the gathered rows and the return of the partial sums (after
        `_gather`, and for the per-pair layout after `_shared_own`)."""
        import torch.distributed as dist
        if self.pairs:
            self._return_pairs(k, valid_local, out_local)
        elif self.fused:
            par = self.step & 1
            self.kernels.forward_scatter_experts(self.x_all, self.valid_all, k, self.dst[par],
                                                 self.rows, self.rank, *self.experts)
            self.handle.barrier(channel=0, timeout_ms=self.timeout_ms)
            self.kernels.reduce_partials(self.slab[par], self.n, self.rows, self.H, valid_local,
                                         out_local)
        else:
            self.kernels.forward_scatter_experts(self.x_all, self.valid_all, k, [self.partial],
                                                 self.n * self.rows, 0, *self.experts)
            dist.reduce_scatter_tensor(self.recv, self.partial, op=dist.ReduceOp.SUM,
                                       group=self.group)
            self.kernels.reduce_partials(self.recv, 1, self.rows, self.H, valid_local, out_local)
        self.step += 1

    def forward(self, x_local, valid_local, k: int, out_local):
        """x_local bf16 [rows, H], valid_local uint8 [rows], out_local bf16 [rows, H]."""
        if self.pairs:
            self._forward_pairs(x_local, valid_local, k, out_local)
            return
        self._gather(x_local, valid_local)
        self._compute_and_return(k, valid_local, out_local)


class TPMoETwoBatch:
    """The two-micro-batch schedule: two TPMoE halves (one per micro-batch, each with
    its own plan, gathered rows and slabs); the all_gather of micro-batch 1 is issued on
    a communication stream so that it runs while micro-batch 0 computes."""

    def __init__(self, full: dict, *, rows: int, **kw):
        (a0, a1), (b0, b1) = split_rows(rows)
        self.ranges = [(a0, a1), (b0, b1)]
        self.halves = [TPMoE(full, rows=a1 - a0, **kw), TPMoE(full, rows=b1 - b0, **kw)]
        self.comm = torch.cuda.Stream(device=full["w_gate_up"].device)

    def forward(self, x_local, valid_local, k: int, out_local):
        main = torch.cuda.current_stream()
        ev = []
        self.comm.wait_stream(main)
        with torch.cuda.stream(self.comm):
            for (lo, hi), half in zip(self.ranges, self.halves):
                half._gather(x_local[lo:hi], valid_local[lo:hi])
                e = torch.cuda.Event()
                e.record(self.comm)
                ev.append(e)
        for e, (lo, hi), half in zip(ev, self.ranges, self.halves):
            half._shared_own(x_local[lo:hi], valid_local[lo:hi])
            main.wait_event(e)
            half._compute_and_return(k, valid_local[lo:hi], out_local[lo:hi])
        main.wait_stream(self.comm)


def pairs_forward_reference(full: dict, x_rows: List[torch.Tensor],
                            valid_rows: List[torch.Tensor], k: int, *, E, H, I, S, Is, fp8,
                            n_shards: int, send_ctas: int = 16):
    """One-GPU emulation of n expert-parallel ranks with the per-pair return (no
    process group): each rank's shared expert on its own rows into its own slab,
    each rank's routed experts sent into every owner's slab, then each owner's
    reduction.  Returns the owners' outputs."""
    dev = full["w_gate_up"].device
    rows = x_rows[0].shape[0]
    x_all = torch.cat(x_rows)
    v_all = torch.cat(valid_rows)
    T = n_shards * rows
    slabs = [torch.full((k + 1, rows, H), float("nan"), dtype=torch.float32, device=dev)
             for _ in range(n_shards)]
    w_all = torch.empty(T, k, dtype=torch.float32, device=dev)
    keep, kerns = [], []
    for r in range(n_shards):
        if S:
            sh = SharedOwnRows(full, H=H, Is=Is, rows=rows, fp8=fp8, device=dev)
            sh.forward(x_rows[r], valid_rows[r], slabs[r][k].data_ptr(), rows)
            keep.append(sh)
        e0, e1 = expert_range(E, n_shards, r)
        shard = {"router_w": full["router_w"], "router_b": full.get("router_b"),
                 "w_gate_up": full["w_gate_up"][e0:e1].contiguous(),
                 "w_down": full["w_down"][e0:e1].contiguous()}
        if fp8:
            shard["s_gate_up"] = full["s_gate_up"][e0:e1].contiguous()
            shard["s_down"] = full["s_down"][e0:e1].contiguous()
        kern = LibraryKernels(shard, E=E, H=H, inter=I, S=0, shared_inter=0, k_max=k, T=T,
                              fp8=fp8, device=dev)
        kern.plan.forward_scatter_pairs(kern.weights, x_all, v_all, k, slabs, rows, k, e0, e1,
                                        send_ctas, dbg=moe.make_debug(topk_w=w_all))
        kerns.append(kern)
        keep.append(shard)
    outs = []
    for r in range(n_shards):
        o = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
        moe.moe_reduce_pairs(slabs[r], k, 1 if S else 0, rows, H, w_all[r * rows:(r + 1) * rows],
                             valid_rows[r], o)
        outs.append(o)
    torch.cuda.synchronize()
    statuses = [kern.plan.device_status() for kern in kerns]
    statuses += [sh.plan.device_status() for sh in keep if isinstance(sh, SharedOwnRows)]
    return outs, statuses


def tp_forward_reference(full: dict, x_rows: List[torch.Tensor], valid_rows: List[torch.Tensor],
                         k: int, *, E, H, I, S, Is, k_max, fp8, n_shards: int, layout: str = "tp"):
    """One-GPU emulation of n ranks (no process group) of either layout: every rank's
    forward scatters into every owner's slab, then each owner reduces.  Returns the
    owners' outputs."""
    dev = full["w_gate_up"].device
    rows = x_rows[0].shape[0]
    x_all = torch.cat(x_rows)
    v_all = torch.cat(valid_rows)
    T = n_shards * rows
    slabs = [torch.full((n_shards, rows, H), float("nan"), dtype=torch.float32, device=dev)
             for _ in range(n_shards)]
    plans = []
    for r in range(n_shards):
        if layout == "tp":
            sh = shard_weights(full, n_shards, r, I=I, Is=Is, fp8=fp8)
            experts, inter = (0, E), I // n_shards
        else:
            sh = shard_experts(full, n_shards, r, E=E, Is=Is, fp8=fp8)
            experts, inter = expert_range(E, n_shards, r), I
        plan = moe.Plan(max_tokens=T, hidden=H, num_experts=E, top_k_max=k_max,
                        inter=inter, num_shared=S, shared_inter=Is // n_shards if S else 0,
                        wtype=moe.MOE_W_FP8_E4M3_B128 if fp8 else moe.MOE_W_BF16, device=dev)
        plan.forward_scatter_experts(make_shard_weights(sh), x_all, v_all, k, [s for s in slabs],
                                     rows, r, *experts)
        plans.append((plan, sh))
    outs = []
    for r in range(n_shards):
        o = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
        moe.moe_reduce_partials(slabs[r], n_shards, rows, H, valid_rows[r], o)
        outs.append(o)
    torch.cuda.synchronize()
    return outs
