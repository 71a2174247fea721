"""Benchmark of the MoE-layer forward pass on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one moe_forward (router, top-k, permute, gather, gate/up GEMM,
down GEMM, combine) over one batch of the workload, inputs resident in HBM.
Prints one JSON line (rank 0).  Under torchrun each rank runs its own batch
(seeded by rank) against the same weights: data-parallel replicas, no
collective on the data path ("scaling": "weak").  --impl reference times the
CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; % of HBM (decode) / tensor-core (prefill) roofline"
DEFAULT_WORKLOAD = "step3_decode"
L2_FLUSH_BYTES = 512 << 20

# DRAM traffic / algorithmic bytes of one gate/up GEMM launch, from the ncu capture
# summarised in profiles/grouped_gemm_step3_e8.md; it applies only to the kernel
# source it was measured on (sha256 prefix), and "traffic" is null otherwise.
GEMM_TRAFFIC = {"sha256_prefix": "0ed45de09043589f", "gate_up_ratio": 0.998}


def gemm_source_hash() -> str:
    import hashlib
    p = os.path.join(ROOT, "mixture_experts_fp32_b200", "csrc", "grouped_gemm.cu")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def launches_per_step(w) -> int:
    """Kernels one forward launches: weight split + router + top-k, the permutation
    (1 kernel up to 1024 rows, 3 above), the row gather (FP8: quantise-and-scatter),
    the two GEMMs and the combine."""
    route = 1 if w.T <= 1024 else 3
    return 3 + route + 1 + 2 + 1


def step_spread(ms) -> dict:
    """Median and 10th / 90th percentiles (linear interpolation) of per-step times."""
    import numpy as np
    if not ms:
        return {"p10": None, "p50": None, "p90": None}
    q = np.percentile(np.asarray(ms, dtype=np.float64), [10, 50, 90])
    return {"p10": float(q[0]), "p50": float(q[1]), "p90": float(q[2])}


def replica_seed(seed: int, rank: int) -> int:
    """Seed of a replica's own batch of hidden states (rank 0 keeps the workload's)."""
    return seed + 1000 * rank


def reduce_over_ranks(v: float, op: str, world: int, device) -> float:
    """max or sum of a per-rank scalar over the process group (identity for 1 rank)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------- algorithmic work

def algorithmic(w, valid_tokens: int, offsets, k: int):
    """Bytes and flops the method must move / compute (touched experts only),
    per step and for the gate/up GEMM alone."""
    import numpy as np
    counts = np.diff(np.asarray(offsets))
    U = int((counts > 0).sum())
    routed_rows = int(counts.sum())
    H, I, E, S, Is = w.H, w.I, w.E, w.S, (w.Is if w.S else 0)
    wb = 2 if w.wtype == "bf16" else 1
    w_gate_up = U * 2 * I * H * wb + S * 2 * Is * H * wb
    w_down = U * H * I * wb + S * H * Is * wb
    router = E * H * 4
    x_read = valid_tokens * H * 2
    out_write = w.T * H * 2
    step_bytes = w_gate_up + w_down + router + x_read + out_write
    expert_flops = 2 * routed_rows * 3 * H * I + 2 * valid_tokens * S * 3 * H * Is
    router_flops = 2 * valid_tokens * E * H
    rows = routed_rows + S * valid_tokens
    gate_up_bytes = w_gate_up + rows * H * 2 + rows * max(I, Is) * 2
    gate_up_flops = 2 * routed_rows * 2 * I * H + 2 * valid_tokens * S * 2 * Is * H
    # the design's intermediates, each written once and read once (not in the
    # roofline): permuted rows x_perm, h, and the expert outputs y
    if w.wtype == "bf16":
        design_bytes = 2 * rows * (H * 2 + max(I, Is) * 2 + H * 4)
    else:   # e4m3 rows with 1x128 fp32 scales, bf16 y
        design_bytes = 2 * rows * (H + H // 128 * 4 + max(I, Is) + max(I, Is) // 128 * 4 + H * 2)
    return {"touched_experts": U, "routed_rows": routed_rows, "step_bytes": step_bytes,
            "step_flops": expert_flops + router_flops, "expert_flops": expert_flops,
            "gate_up_bytes": gate_up_bytes, "gate_up_flops": gate_up_flops,
            "design_bytes": design_bytes}


# ------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3])
                          if v.lower() == "active"})
        loaded = [r[0] for r in rows if r[2] > 200.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ our arm

def run_native(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import mixture_experts_fp32_b200 as moe
    from mixture_experts_fp32_b200.pipeline import HostPipeline
    from mixture_experts_fp32_b200 import build as lib_build
    import synth

    ws_n, rank, local = dist_env()
    if ws_n > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=600))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    if rank == 0:
        lib_build.build()
    if ws_n > 1:
        dist.barrier()
    moe.load()

    w = workload_of(args)
    k = w.k
    # weights: drawn once (rank 0) and broadcast; activations: one batch per rank
    inp = synth.make_inputs(w, with_weights=(rank == 0))
    if ws_n > 1:
        inp["x"] = synth.normal_bf16(replica_seed(w.seed, rank), synth.STREAM_X, (w.T, w.H),
                                     w.x_sigma)
    d = {}
    for key in ("x", "valid", "router_w", "router_b"):
        d[key] = None if inp.get(key) is None else inp[key].to(dev)
    wkeys = ["w_gate_up", "w_down", "ws_gate_up", "ws_down", "s_gate_up", "s_down",
             "ss_gate_up", "ss_down"]
    for key in wkeys:
        if rank == 0:
            d[key] = None if inp.get(key) is None else inp[key].to(dev)
    if ws_n > 1:
        shapes = [None if d.get(kk) is None else (tuple(d[kk].shape), d[kk].dtype)
                  for kk in wkeys] if rank == 0 else None
        obj = [shapes]
        dist.broadcast_object_list(obj, src=0)
        shapes = obj[0]
        for kk, sh in zip(wkeys, shapes):
            if sh is None:
                d[kk] = None
                continue
            if rank != 0:
                d[kk] = torch.empty(sh[0], dtype=sh[1], device=dev)
            dist.broadcast(d[kk], src=0)
    del inp

    plan = moe.Plan(max_tokens=w.T, hidden=w.H, num_experts=w.E, top_k_max=k, inter=w.I,
                    num_shared=w.S, shared_inter=w.Is if w.S else 0, device=dev,
                    wtype=moe.MOE_W_BF16 if w.wtype == "bf16" else moe.MOE_W_FP8_E4M3_B128)
    weights = plan.weights(d["router_w"], d["router_b"], d["w_gate_up"], d["w_down"],
                           d.get("s_gate_up"), d.get("s_down"), d.get("ws_gate_up"),
                           d.get("ws_down"), d.get("ss_gate_up"), d.get("ss_down"))
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    offsets = torch.empty(w.E + 1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    valid_tokens = int(d["valid"].sum().item())

    def fwd(events=None, want_offsets=False):
        dbg = moe.make_debug(offsets=offsets if want_offsets else None, events=events)
        plan.forward(weights, d["x"], d["valid"], k, out, stream=stream, dbg=dbg)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        fwd(want_offsets=True)
    torch.cuda.synchronize()
    if plan.device_status() != 0:
        raise RuntimeError("device status set during warm-up")
    algo = algorithmic(w, valid_tokens, offsets.cpu().numpy(), k)

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.MOE_NUM_STAGES + 1)]
          for _ in range(K)]
    # torch creates the CUDA event on first record; the library records them again in-step
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    # nvidia-smi samples every 200 ms and the timed steps take milliseconds, so the
    # sampler also covers ~1.5 s of further (untimed) warm-up steps right before them
    clocks = ClockSampler(dev.index)
    clocks.start()
    t_end = time.perf_counter() + 1.5
    while time.perf_counter() < t_end:
        for _ in range(8):
            flush.zero_()
            fwd()
        torch.cuda.synchronize()
    if ws_n > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    for i in range(K):
        flush.zero_()                      # L2 flush outside the step's events
        fwd(events=ev[i])
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    clock_info = clocks.stop()
    if ws_n > 1:
        dist.barrier()
    step_ms = [ev[i][0].elapsed_time(ev[i][moe.MOE_NUM_STAGES]) for i in range(K)]
    stage_ms = {name: statistics.mean(ev[i][s].elapsed_time(ev[i][s + 1]) for i in range(K))
                for s, name in enumerate(moe.STAGE_NAMES)}
    status = plan.device_status()
    total_ms = sum(step_ms)
    gemm_ms = stage_ms["gate_up_gemm"]

    # the same step replayed from a CUDA graph captured once (outside the timed region)
    graph_ms = None
    if args.graph:
        out_g = torch.empty_like(out)
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            plan.forward(weights, d["x"], d["valid"], k, out_g, stream=cap)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        if ws_n > 1:
            dist.barrier()
        torch.cuda.synchronize()
        gms = []
        for _ in range(K):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            e1.synchronize()
            gms.append(e0.elapsed_time(e1))
        torch.cuda.synchronize()
        if ws_n > 1:
            dist.barrier()
        if not torch.equal(out_g.view(torch.int16), out.view(torch.int16)):
            raise RuntimeError("graph replay differs from the eager forward")
        graph_ms = reduce_over_ranks(sum(gms), "max", ws_n, dev) / K
        del g

    # end to end: pinned host input -> device, forward, result -> pinned host.
    # Serial: each step's copies and forward one after another on one stream.
    x_host = d["x"].cpu().pin_memory()
    v_host = d["valid"].cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    x_dev = torch.empty_like(d["x"])
    v_dev = torch.empty_like(d["valid"])
    for _ in range(2):
        x_dev.copy_(x_host, non_blocking=True)
        v_dev.copy_(v_host, non_blocking=True)
        plan.forward(weights, x_dev, v_dev, k, out, stream=stream)
        out_host.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    e2e_ms = []
    for _ in range(K):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        x_dev.copy_(x_host, non_blocking=True)
        v_dev.copy_(v_host, non_blocking=True)
        plan.forward(weights, x_dev, v_dev, k, out, stream=stream)
        out_host.copy_(out, non_blocking=True)
        e1.record()
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))

    # Pipelined (the headline e2e): HostPipeline runs every step's upload and
    # download on copy streams beside the neighbouring steps' forwards; K steps
    # back to back, timed from before the first upload to after the last download
    pipe = HostPipeline(plan, weights, k, w.T, depth=3, graph=args.graph)
    outs_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(3)]
    for i in range(3):
        pipe.submit(x_host, v_host, outs_host[i % 3])
    pipe.synchronize()
    if ws_n > 1:
        dist.barrier()
    torch.cuda.synchronize()
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(pipe.up)
    for i in range(K):
        pipe.submit(x_host, v_host, outs_host[i % 3])
    p1.record(pipe.down)
    p1.synchronize()
    pipe_ms = p0.elapsed_time(p1)
    pipe.close()
    if not torch.equal(outs_host[(K - 1) % 3].view(torch.int16), out.cpu().view(torch.int16)):
        raise RuntimeError("pipelined output differs from the eager forward")

    total_ms = reduce_over_ranks(total_ms, "max", ws_n, dev)
    e2e_total = reduce_over_ranks(sum(e2e_ms), "max", ws_n, dev)
    pipe_total = reduce_over_ranks(pipe_ms, "max", ws_n, dev)
    tokens = reduce_over_ranks(float(valid_tokens), "sum", ws_n, dev)
    status = int(reduce_over_ranks(float(status), "max", ws_n, dev))

    peaks = measured_peaks()
    prefill = w.wtype == "fp8"
    bound = "tensor" if prefill else "hbm"
    if bound == "hbm":
        achieved = algo["gate_up_bytes"] / (gemm_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    else:
        achieved = algo["gate_up_flops"] / (gemm_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"] * (2 if w.wtype == "fp8" else 1)
        unit = "TFLOP/s"
    traffic = None
    if gemm_source_hash() == GEMM_TRAFFIC["sha256_prefix"] and w.wtype == "bf16":
        traffic = GEMM_TRAFFIC["gate_up_ratio"] * algo["gate_up_bytes"]
    ms = total_ms / K
    # expert flops at the weights' dtype peak (FP8: twice the measured bf16 figure,
    # the nominal dense ratio), router flops (fp32 logits) at the bf16 figure
    mm_peak = peaks["bf16_tflops"] * (2 if w.wtype == "fp8" else 1) * 1e12
    step_roof_ms = max(algo["step_bytes"] / (peaks["hbm_gbs"] * 1e9),
                       algo["expert_flops"] / mm_peak
                       + (algo["step_flops"] - algo["expert_flops"]) / (peaks["bf16_tflops"] * 1e12)
                       ) * 1e3

    result = None
    if rank == 0:
        cpu = cpu_baseline(w, args) if (ws_n == 1 and not args.no_cpu_baseline) else None
        # headline: the step replayed from a CUDA graph (how a serving engine runs a
        # decode step); the eager pass gives the per-stage breakdown and kernel times
        head_ms = graph_ms if graph_ms is not None else ms
        result = {
            "metric": METRIC, "value": tokens / (head_ms * 1e-3) if K else 0.0,
            "unit": "tokens/s", "n_gpus": ws_n, "steps": K, "warmup": max(args.warmup, 3),
            "ms_per_step": head_ms, "higher_is_better": True, "scaling": "weak",
            "timing": ("CUDA-graph replay of one captured forward per step"
                       if graph_ms is not None else "eager forward per step"),
            "eager": {"ms_per_step": ms, "value": tokens / (ms * 1e-3)},
            "vs_baseline": None, "dtype": w.wtype, "data": "synthetic (Philox4x32-10, seed 0)",
            "config": {"workload": w.name, "T": w.T, "valid_tokens": valid_tokens, "H": w.H,
                       "E": w.E, "k": k, "I": w.I, "S": w.S, "Is": w.Is,
                       "parallelism": f"dp{ws_n} replicas" if ws_n > 1 else "single GPU",
                       "l2": f"{L2_FLUSH_BYTES >> 20} MB written between timed steps, "
                             "outside the step events; weights alone exceed L2"},
            "roofline": {"bound": bound, "kernel": "grouped_gemm gate/up + SwiGLU",
                         "achieved": achieved, "peak": peak, "unit": unit,
                         "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_bytes": algo["gate_up_bytes"],
                         "algorithmic_flops": algo["gate_up_flops"],
                         "launch_ms": gemm_ms, "peak_source": peaks["source"],
                         # the same kernel against the matmul rate measured over seconds
                         # under the power cap (the timed steps run back to back)
                         "frac_of_sustained": (achieved / (peaks["bf16_tflops_sustained"]
                                                           * (2 if w.wtype == "fp8" else 1))
                                               if bound == "tensor"
                                               and peaks.get("bf16_tflops_sustained")
                                               else None)},
            "step_roofline": {"ms": step_roof_ms, "frac": step_roof_ms / head_ms,
                              "frac_eager": step_roof_ms / ms,
                              "algorithmic_bytes": algo["step_bytes"],
                              "algorithmic_flops": algo["step_flops"],
                              "touched_experts": algo["touched_experts"],
                              "design_bytes": algo["design_bytes"],
                              "design_ms_at_hbm": algo["design_bytes"]
                              / (peaks["hbm_gbs"] * 1e9) * 1e3},
            "stage_ms": stage_ms,
            "step_ms_spread": {"rank": 0, "eager": step_spread(step_ms),
                               "graph": step_spread(gms) if graph_ms is not None else None,
                               "e2e_serial": step_spread(e2e_ms)},
            "e2e": {"value": tokens / (pipe_total * 1e-3 / K), "unit": "tokens/s",
                    "ms_per_step": pipe_total / K,
                    "h2d_bytes_per_step": x_host.numel() * 2 + v_host.numel(),
                    "d2h_bytes_per_step": out_host.numel() * 2,
                    "how": "the library's host-to-host pipeline (moe_pipeline_*, C ABI with "
                           "host buffers): K steps back to back, each uploading its x and mask "
                           "from pinned host memory and downloading its output to pinned host "
                           "memory on copy streams beside the neighbouring steps' forwards "
                           "(3 slots" + (", graph replay" if args.graph else "") + "); L2 not "
                           "flushed: every step streams its weights (far above L2) through it"},
            "e2e_serial": {"value": tokens / (e2e_total * 1e-3 / K), "unit": "tokens/s",
                           "ms_per_step": e2e_total / K,
                           "how": "upload, eager forward and download one after another on "
                                  "one stream, L2 flushed before each step"},
            "gpu_launches": launches_per_step(w) * K,
            "graph_replay": None if graph_ms is None else {
                "ms_per_step": graph_ms, "value": tokens / (graph_ms * 1e-3),
                "unit": "tokens/s"},
            "clocks": clock_info,
            "device_status": status,
            "wall_s_timed_region": t_wall,
            "cpu_baseline": cpu,
        }
        print(json.dumps(result), flush=True)
    if ws_n > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# --------------------------------------------------------- the CPU oracle

def oracle_tokens_per_s(w, target_s: float):
    """Times the oracle (routing and expert FFN) on growing samples of the
    workload's valid tokens until one sample takes about target_s seconds."""
    import numpy as np

    import oracle
    import synth
    inp = synth.make_inputs(w)
    valid_idx = np.nonzero(inp["valid"].numpy())[0]
    cores = oracle.max_threads()          # the threads the oracle's loops actually use
    n = min(len(valid_idx), max(1, cores))
    while True:
        tok = valid_idx[:n]
        t0 = time.perf_counter()
        sub = dict(inp)
        sub["x"] = inp["x"][tok]
        sub["valid"] = inp["valid"][tok]
        logits = oracle.router_logits(sub["x"], sub["valid"], inp["router_w"], inp["router_b"])
        ids, wt = oracle.topk(logits, sub["valid"], w.k)
        oracle.route(ids, sub["valid"], w.E)
        oracle.moe_tokens(sub, ids, wt)
        dt = time.perf_counter() - t0
        if dt >= target_s / 4 or n >= len(valid_idx):
            return n / dt, n, dt, cores
        n = min(len(valid_idx), int(n * max(2.0, target_s / max(dt, 1e-3))))


def cpu_baseline(w, args):
    rate, n, dt, cores = oracle_tokens_per_s(w, args.cpu_seconds)
    return {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} valid tokens of {w.name} (all weights), {dt:.1f} s, "
                      f"double-precision C with OpenMP over tokens"}


def run_tp(args):
    """Tensor- or expert-parallel layout (--tp, --tp-layout tp|ep): the workload's rows
    are the all-gathered batch of N DP ranks (rows T/N each); every rank holds 1/N of
    each expert's intermediate dimension (tp) or 1/N of the experts and of the shared
    expert (ep) and returns its partial sums to the owners (fused into the combine, or
    NCCL reduce_scatter with --tp-return nccl).  Whole-job valid tokens/s; the gathered
    batch is fixed, so adding ranks is strong scaling."""
    import socket

    import torch
    import torch.distributed as dist

    import mixture_experts_fp32_b200 as moe
    from mixture_experts_fp32_b200 import build as lib_build
    from mixture_experts_fp32_b200 import tp
    import synth

    ws_n, rank, local = dist_env()
    if "MASTER_ADDR" not in os.environ:                   # one process without torchrun
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(sk.getsockname()[1]))
        sk.close()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", rank=rank, world_size=ws_n, device_id=dev,
                            timeout=__import__("datetime").timedelta(seconds=600))
    layer = None
    try:
        if rank == 0:
            lib_build.build()
        dist.barrier()
        moe.load()
        w = workload_of(args)
        if w.T % ws_n:
            raise SystemExit(f"{w.T} rows do not split over {ws_n} ranks")
        rows = w.T // ws_n
        inp = synth.make_inputs(w)        # the same seeded layer and gathered batch on every rank
        d = {key: (v.to(dev) if isinstance(v, torch.Tensor) else v) for key, v in inp.items()}
        del inp
        layer = tp.TPMoE(d, E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is if w.S else 0, k_max=w.k,
                         rows=rows, fp8=w.wtype == "fp8", fused=args.tp_return == "fused",
                         layout=args.tp_layout)
        x_loc = d["x"][rank * rows:(rank + 1) * rows].contiguous()
        v_loc = d["valid"][rank * rows:(rank + 1) * rows].contiguous()
        valid_tokens = int(d["valid"].sum().item())
        for key in ("w_gate_up", "w_down", "ws_gate_up", "ws_down", "s_gate_up", "s_down",
                    "ss_gate_up", "ss_down"):
            d[key] = None                                  # the shard keeps its own copy
        torch.cuda.empty_cache()
        out = torch.empty(rows, w.H, dtype=torch.bfloat16, device=dev)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            layer.forward(x_loc, v_loc, w.k, out)
        torch.cuda.synchronize()
        if layer.plan.device_status() != 0:
            raise RuntimeError("device status set during warm-up")
        K = args.steps
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        clocks = ClockSampler(dev.index)
        clocks.start()
        dist.barrier()
        torch.cuda.synchronize()
        for e0, e1 in ev:
            flush.zero_()
            e0.record()
            layer.forward(x_loc, v_loc, w.k, out)
            e1.record()
        torch.cuda.synchronize()
        dist.barrier()
        clk = clocks.stop()
        ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / K
        ms = reduce_over_ranks(ms, "max", ws_n, dev)
        if layer.plan.device_status() != 0:
            raise RuntimeError("device status set during the timed steps")
        if rank == 0:
            print(json.dumps({
                "metric": METRIC, "value": valid_tokens / (ms * 1e-3), "unit": "tokens/s",
                "n_gpus": ws_n, "steps": K, "warmup": max(args.warmup, 3), "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": w.wtype, "data": "synthetic (Philox4x32-10, seed 0)",
                "timing": "eager TP forward per step (all_gather, layer, partial return, reduce)",
                "config": {"workload": w.name, "T": w.T, "valid_tokens": valid_tokens,
                           "rows_per_rank": rows, "H": w.H, "E": w.E, "k": w.k, "I": w.I,
                           "S": w.S, "parallelism": f"{args.tp_layout}{ws_n}",
                           "partial_return": args.tp_return,
                           "l2": f"{L2_FLUSH_BYTES >> 20} MB written between timed steps"},
                "clocks": clk}))
    finally:
        del layer
        torch.cuda.synchronize()
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    ws_n, rank, _ = dist_env()
    if rank != 0:
        return None
    w = workload_of(args)
    rates = []
    for _ in range(max(args.warmup, 0)):
        oracle_tokens_per_s(w, min(args.cpu_seconds, 5.0))
    n = dt = cores = 0
    for _ in range(args.steps):
        r, n, dt, cores = oracle_tokens_per_s(w, args.cpu_seconds)
        rates.append(r)
    value = statistics.median(rates) if rates else 0.0
    res = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * n / value if value else 0,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (Philox4x32-10, seed 0)", "impl": "reference",
           "config": {"workload": w.name, "T": w.T, "H": w.H, "E": w.E, "k": w.k, "I": w.I,
                      "S": w.S, "Is": w.Is},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                            "kind": "oracle",
                            "sample": f"{n} valid tokens per step of {w.name}, {dt:.1f} s"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)
    return res


def workload_of(args):
    import synth
    w = synth.WORKLOADS[args.workload]
    if args.experts:
        # a smaller copy of the workload (fewer experts) for profiler captures
        w = w.with_(name=f"{w.name}_e{args.experts}", E=args.experts, k=min(w.k, args.experts))
    return w


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time eager forwards only (default: the headline is CUDA-graph replay)")
    ap.add_argument("--tp", action="store_true",
                    help="tensor-parallel layout over the N ranks (default workload: dp_padded)")
    ap.add_argument("--tp-return", default="fused", choices=["fused", "nccl"])
    ap.add_argument("--tp-layout", default="tp", choices=["tp", "ep"],
                    help="with --tp: split every expert's intermediate dimension (tp) or "
                         "the experts (ep) over the ranks")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the number of routed experts (profiling on a smaller case)")
    args = ap.parse_args(argv)
    if args.tp and args.workload == DEFAULT_WORKLOAD and "--workload" not in (argv or sys.argv):
        args.workload = "dp_padded"
    if args.impl == "reference":
        run_reference(args)
    elif args.tp:
        run_tp(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
