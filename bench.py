"""Benchmark of the MoE-layer forward pass on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one moe_forward (router, top-k, permute, gather, gate/up GEMM,
down GEMM, combine) over one batch of the workload, inputs resident in HBM.
Prints one JSON line (rank 0).  On one GPU the line is the Step3 decode step
(the headline) and carries the other timed workloads (DeepSeek-style decode,
the DP-padded gather batch, FP8 block-scale prefill) under "workloads", each
measured the same way in the same run; --workload NAME times that one alone.
Under torchrun (N > 1) the default is the tensor-parallel layer behind DP
attention on the Step3 decode batch (all_gather of the ranks' rows, every
rank 1/N of each expert's intermediate dimension, partial sums returned into
the owners' slabs by the combine): strong scaling of the same batch.
--replicas runs N independent data-parallel replicas instead.  --impl
reference times the CPU oracle on the host cores instead.
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
# the default one-GPU run: the headline first, then the other timed workloads
ALL_WORKLOADS = ("step3_decode", "deepseek_decode", "dp_padded", "fp8_prefill")
L2_FLUSH_BYTES = 512 << 20

# DRAM traffic / algorithmic bytes of one bf16 gate/up GEMM launch, from an ncu
# capture of that kernel on the Step3 decode shape (8 experts, 1 GPU); it applies
# only to the kernel source it was measured on (sha256 prefix), and "traffic" is
# null otherwise.
GEMM_TRAFFIC = {"sha256_prefix": "5a12df72098ca22e", "gate_up_ratio": 1.000}


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


def _time_loop(fn, burst_reps: int = 10, sustain_s: float = 3.0):
    """Best single-call time over burst_reps calls, and the mean time per call of
    calls issued back to back for about sustain_s seconds (CUDA events, ms)."""
    import torch
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(burst_reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1))
    n = max(8, int(sustain_s * 1e3 / max(best, 1e-3)))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        fn()
    e1.record()
    e1.synchronize()
    return best, e0.elapsed_time(e1) / n


def measure_fp8_peak(n: int = 8192, sustain_s: float = 3.0) -> dict:
    """Dense e4m3 tensor-core rate on this GPU, measured with the library GEMM of
    the framework (cuBLASLt through torch): an n^3 e4m3 x e4m3 -> bf16 product with
    one fp32 scale per tensor, best of 10 (burst) and back to back for sustain_s
    (sustained).  The same product with 1x128 activation and 128x128 weight block
    scales (the layer's arithmetic) is timed beside it where torch offers it."""
    import torch
    import torch.nn.functional as F
    g = torch.Generator(device="cuda").manual_seed(0)
    a = (torch.randn(n, n, device="cuda", generator=g) * 0.5).to(torch.float8_e4m3fn)
    bt = (torch.randn(n, n, device="cuda", generator=g) * 0.5).to(torch.float8_e4m3fn)
    one = torch.ones((), device="cuda", dtype=torch.float32)
    flops = 2.0 * n ** 3
    res = {"shape": f"{n}x{n}x{n} e4m3 -> bf16", "how": "torch._scaled_mm (cuBLASLt)"}
    best, sus = _time_loop(lambda: torch._scaled_mm(a, bt.t(), one, one,
                                                    out_dtype=torch.bfloat16), sustain_s=sustain_s)
    res["tensorwise_tflops"] = flops / (best * 1e-3) / 1e12
    res["tensorwise_tflops_sustained"] = flops / (sus * 1e-3) / 1e12
    try:
        kb = n // 128
        sa = torch.rand(kb, n, device="cuda", generator=g).add_(0.5).t()      # [n, n/128]
        l4 = (kb + 3) // 4 * 4
        sb = torch.rand(n // 128, l4, device="cuda", generator=g).add_(0.5).t()  # [l4, n/128]
        ST, SW = F.ScalingType, F.SwizzleType

        def blockwise():
            return F.scaled_mm(a, bt.t(), [sa], [ST.BlockWise1x128], [sb],
                               [ST.BlockWise128x128], [SW.NO_SWIZZLE], [SW.NO_SWIZZLE],
                               None, torch.bfloat16)
        best, sus = _time_loop(blockwise, sustain_s=min(sustain_s, 1.0))
        res["blockwise_1x128_128x128_tflops"] = flops / (best * 1e-3) / 1e12
        res["blockwise_1x128_128x128_tflops_sustained"] = flops / (sus * 1e-3) / 1e12
    except Exception as ex:   # not offered by this torch / cuBLASLt build
        res["blockwise_1x128_128x128_tflops"] = None
        res["blockwise_error"] = f"{type(ex).__name__}: {str(ex)[:160]}"
    del a, bt
    torch.cuda.empty_cache()
    return res


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def launches_per_step(w) -> int:
    """Kernels one forward launches: router + top-k, the permutation (1 kernel up to
    1024 rows, 3 above), the row gather (FP8: quantise-and-scatter), the two GEMMs
    and the combine.  The router weights' bf16 split is made once with the weights
    (moe_split_router_weights), not per step."""
    route = 1 if w.T <= 1024 else 3
    return 2 + route + 1 + 2 + 1


def tp_launches_per_step(w, n_ranks: int, rows: int, n_mb: int, ret: str) -> int:
    """This library's kernels one step of the tensor- / expert-parallel layer launches
    (NCCL's and the symmetric-memory barrier's not counted): per micro-batch the
    layer over the gathered rows and the owner's reduction; with the per-pair return
    the combine is replaced by the sends inside the down GEMM, and the shared expert
    runs on the rank's own rows as a one-expert layer (router, top-k, one route
    kernel, gather, two GEMMs, combine)."""
    total = 0
    for lo, hi in ([(0, rows // 2), (rows // 2, rows)] if n_mb == 2 else [(0, rows)]):
        layer = launches_per_step(w.with_(T=n_ranks * (hi - lo)))
        if ret == "pairs":
            total += (layer - 1) + 1 + (7 if w.S else 0)
        else:
            total += layer + 1
    return total


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
    if w.wtype == "bf16":      # bf16 x_perm, h in two bf16 parts, fp32 y
        design_bytes = 2 * rows * (H * 2 + max(I, Is) * 4 + H * 4)
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

def setup_dist(ws_n: int, local: int):
    import datetime

    import torch
    import torch.distributed as dist
    if ws_n > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=datetime.timedelta(seconds=600))
    else:
        torch.cuda.set_device(0)
    return torch.device("cuda", torch.cuda.current_device())


def expert_load(offsets) -> dict:
    """The realised routing: rows per routed expert (pairs), summarised."""
    import numpy as np
    c = np.diff(np.asarray(offsets, dtype=np.int64))
    t = c[c > 0]
    if t.size == 0:
        return {"touched": 0}
    return {"touched": int(t.size), "pairs": int(c.sum()), "max_rows": int(t.max()),
            "min_rows_touched": int(t.min()), "mean_rows_touched": float(t.mean()),
            "cv_touched": float(t.std() / t.mean()),
            "top8_share": float(np.sort(c)[::-1][:8].sum() / max(1, c.sum()))}


def run_native(args):
    """One GPU (or --replicas: N data-parallel replicas, no collective on the data
    path): every workload of the run measured in turn, the first one the headline."""
    import torch
    import torch.distributed as dist

    import mixture_experts_fp32_b200 as moe
    from mixture_experts_fp32_b200 import build as lib_build

    ws_n, rank, local = dist_env()
    dev = setup_dist(ws_n, local)
    if rank == 0:
        lib_build.build()
    if ws_n > 1:
        dist.barrier()
    moe.load()
    peaks = measured_peaks()
    names = [args.workload] if args.single else list(ALL_WORKLOADS)
    fp8_peak = None
    results = {}
    for i, name in enumerate(names):
        w = workload_of(args, name)
        if w.wtype == "fp8" and fp8_peak is None and not args.no_fp8_peak:
            fp8_peak = measure_fp8_peak()
            fp8_peak = {kk: (reduce_over_ranks(v, "max", ws_n, dev)
                             if isinstance(v, float) else v) for kk, v in fp8_peak.items()}
        results[name] = measure_workload(args, w, dev, ws_n, rank, peaks, fp8_peak,
                                         headline=(i == 0))
        torch.cuda.empty_cache()
    result = None
    if rank == 0:
        result = results[names[0]]["line"]
        if len(names) > 1:
            result["workloads"] = {n: results[n]["summary"] for n in names}
        result["fp8_peak"] = fp8_peak
        print(json.dumps(result), flush=True)
    if ws_n > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def measure_workload(args, w, dev, ws_n, rank, peaks, fp8_peak, headline: bool):
    """Times one workload: eager steps with the library's stage events, the same
    step replayed from a CUDA graph (the headline time), and for the headline the
    end-to-end host-to-host figure; then the CPU-baseline leg (rank 0, one GPU),
    which also reports the parity of sampled rows against the oracle."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import mixture_experts_fp32_b200 as moe
    from mixture_experts_fp32_b200.pipeline import HostPipeline
    import synth

    k = w.k
    t_gen = time.perf_counter()
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
    # the host copies the oracle leg needs (hidden states, mask, router; the
    # weights it reads are these same tensors)
    host = inp if (rank == 0 and ws_n == 1) else None
    del inp
    t_gen = time.perf_counter() - t_gen

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
        raise RuntimeError(f"{w.name}: device status set during warm-up")
    off_host = offsets.cpu().numpy()
    algo = algorithmic(w, valid_tokens, off_host, k)

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

    # the same step replayed from a CUDA graph captured once (outside the timed region)
    graph_ms = None
    gms = []
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
            raise RuntimeError(f"{w.name}: graph replay differs from the eager forward")
        graph_ms = reduce_over_ranks(sum(gms), "max", ws_n, dev) / K
        del g
    clock_info = clocks.stop()
    if ws_n > 1:
        dist.barrier()
    step_ms = [ev[i][0].elapsed_time(ev[i][moe.MOE_NUM_STAGES]) for i in range(K)]
    stage_ms = {name: statistics.mean(ev[i][s].elapsed_time(ev[i][s + 1]) for i in range(K))
                for s, name in enumerate(moe.STAGE_NAMES)}
    status = plan.device_status()
    total_ms = reduce_over_ranks(sum(step_ms), "max", ws_n, dev)
    gemm_ms = stage_ms["gate_up_gemm"]

    e2e = e2e_serial = e2e_ms = None
    if headline:
        e2e, e2e_serial, e2e_ms = end_to_end(args, w, d, plan, weights, out, k, flush, stream,
                                             valid_tokens, ws_n, dev, HostPipeline)

    # routing and outputs of this batch for the parity leg (one more forward)
    gpu = None
    if host is not None and not args.no_cpu_baseline:
        dbg_t = {"logits": torch.empty(w.T, w.E, dtype=torch.float32, device=dev),
                 "topk_ids": torch.empty(w.T, k, dtype=torch.int32, device=dev),
                 "topk_w": torch.empty(w.T, k, dtype=torch.float32, device=dev)}
        plan.forward(weights, d["x"], d["valid"], k, out, stream=stream,
                     dbg=moe.make_debug(**dbg_t))
        torch.cuda.synchronize()
        gpu = {key: v.cpu() for key, v in dbg_t.items()}
        gpu["out"] = out.cpu()
    del d, weights, plan, flush, out
    torch.cuda.empty_cache()

    status = int(reduce_over_ranks(float(status), "max", ws_n, dev))
    tokens = reduce_over_ranks(float(valid_tokens), "sum", ws_n, dev)
    if rank != 0:
        return None
    fp8 = w.wtype == "fp8"
    bound = "tensor" if fp8 else "hbm"
    if fp8 and fp8_peak is not None:
        mm_peak = fp8_peak["tensorwise_tflops"]
        mm_sustained = fp8_peak["tensorwise_tflops_sustained"]
        peak_source = "measured_fp8 (e4m3 GEMM of the same run, burst)"
    elif fp8:
        mm_peak = 2 * peaks["bf16_tflops"]
        mm_sustained = 2 * (peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"])
        peak_source = "2x measured bf16 (nominal dense ratio)"
    else:
        mm_peak = peaks["bf16_tflops"]
        mm_sustained = peaks["bf16_tflops_sustained"]
        peak_source = peaks["source"]
    if bound == "hbm":
        achieved = algo["gate_up_bytes"] / (gemm_ms * 1e-3) / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
        frac_sus = None
    else:
        achieved = algo["gate_up_flops"] / (gemm_ms * 1e-3) / 1e12
        peak, unit = mm_peak, "TFLOP/s"
        frac_sus = achieved / mm_sustained if mm_sustained else None
    traffic = None
    if gemm_source_hash() == GEMM_TRAFFIC["sha256_prefix"] and not fp8:
        traffic = GEMM_TRAFFIC["gate_up_ratio"] * algo["gate_up_bytes"]
    ms = total_ms / K
    # expert flops at the weights' dtype peak, router flops (fp32 logits on the
    # bf16 tensor path) at the bf16 figure
    step_roof_ms = max(algo["step_bytes"] / (peaks["hbm_gbs"] * 1e9),
                       algo["expert_flops"] / (mm_peak * 1e12)
                       + (algo["step_flops"] - algo["expert_flops"]) / (peaks["bf16_tflops"] * 1e12)
                       ) * 1e3
    head_ms = graph_ms if graph_ms is not None else ms
    cpu = None
    if host is not None and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, host, gpu, args.cpu_seconds if headline else args.parity_seconds)
    roofline = {"bound": bound, "kernel": ("grouped_gemm_fp8 gate/up + SwiGLU + h quantisation"
                                           if fp8 else "grouped_gemm gate/up + SwiGLU"),
                "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": traffic, "algorithmic_bytes": algo["gate_up_bytes"],
                "algorithmic_flops": algo["gate_up_flops"], "launch_ms": gemm_ms,
                "peak_source": peak_source if bound == "tensor" else peaks["source"],
                # the same kernel against the rate measured over seconds under the
                # power cap (the timed steps run back to back)
                "frac_of_sustained": frac_sus}
    step_roof = {"ms": step_roof_ms, "frac": step_roof_ms / head_ms,
                 "frac_eager": step_roof_ms / ms,
                 "algorithmic_bytes": algo["step_bytes"], "algorithmic_flops": algo["step_flops"],
                 "touched_experts": algo["touched_experts"],
                 "design_bytes": algo["design_bytes"],
                 "design_ms_at_hbm": algo["design_bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e3}
    config = {"workload": w.name, "T": w.T, "valid_tokens": valid_tokens, "H": w.H, "E": w.E,
              "k": k, "I": w.I, "S": w.S, "Is": w.Is, "wtype": w.wtype,
              "parallelism": f"dp{ws_n} replicas" if ws_n > 1 else "single GPU",
              "l2": f"{L2_FLUSH_BYTES >> 20} MB written between timed steps, outside the "
                    "step events; weights alone exceed L2"}
    summary = {"ms_per_step": head_ms, "value": tokens / (head_ms * 1e-3), "unit": "tokens/s",
               "eager_ms_per_step": ms, "timing": ("CUDA-graph replay" if graph_ms is not None
                                                   else "eager"),
               "config": config, "roofline": roofline, "step_roofline": step_roof,
               "stage_ms": stage_ms, "clocks": clock_info,
               "step_ms_spread": {"eager": step_spread(step_ms),
                                  "graph": step_spread(gms) if gms else None},
               "expert_load": expert_load(off_host),
               "parity": None if cpu is None else cpu.get("parity"),
               "gpu_launches": launches_per_step(w) * K, "device_status": status,
               "input_generation_s": t_gen}
    line = {
        "metric": METRIC, "value": tokens / (head_ms * 1e-3) if K else 0.0,
        "unit": "tokens/s", "n_gpus": ws_n, "steps": K, "warmup": max(args.warmup, 3),
        "ms_per_step": head_ms, "higher_is_better": True, "scaling": "weak",
        "timing": ("CUDA-graph replay of one captured forward per step"
                   if graph_ms is not None else "eager forward per step"),
        "eager": {"ms_per_step": ms, "value": tokens / (ms * 1e-3)},
        "vs_baseline": None, "dtype": w.wtype, "data": "synthetic (Philox4x32-10, seed 0)",
        "config": config, "roofline": roofline, "step_roofline": step_roof,
        "stage_ms": stage_ms,
        "step_ms_spread": {"rank": 0, "eager": step_spread(step_ms),
                           "graph": step_spread(gms) if gms else None,
                           "e2e_serial": step_spread(e2e_ms) if e2e_ms else None},
        "e2e": e2e, "e2e_serial": e2e_serial,
        "gpu_launches": launches_per_step(w) * K,
        "graph_replay": None if graph_ms is None else {
            "ms_per_step": graph_ms, "value": tokens / (graph_ms * 1e-3), "unit": "tokens/s"},
        "clocks": clock_info, "device_status": status, "wall_s_timed_region": t_wall,
        "expert_load": summary["expert_load"],
        "parity": summary["parity"],
        "cpu_baseline": cpu,
    }
    return {"line": line, "summary": summary}


def end_to_end(args, w, d, plan, weights, out, k, flush, stream, valid_tokens, ws_n, dev,
               HostPipeline):
    """The step through the C ABI with host buffers: pinned host input -> device,
    forward, result -> pinned host.  Serial: each step's copies and forward one
    after another on one stream; pipelined (the e2e headline): the library's
    host-to-host pipeline, copies on its own streams beside the neighbouring
    steps' forwards."""
    import torch
    import torch.distributed as dist
    K = args.steps
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

    # K steps back to back, timed from before the first upload to after the last download
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
    e2e_total = reduce_over_ranks(sum(e2e_ms), "max", ws_n, dev)
    pipe_total = reduce_over_ranks(pipe_ms, "max", ws_n, dev)
    tokens = reduce_over_ranks(float(valid_tokens), "sum", ws_n, dev)
    e2e = {"value": tokens / (pipe_total * 1e-3 / K), "unit": "tokens/s",
           "ms_per_step": pipe_total / K,
           "h2d_bytes_per_step": x_host.numel() * 2 + v_host.numel(),
           "d2h_bytes_per_step": out_host.numel() * 2,
           "how": "the library's host-to-host pipeline (moe_pipeline_*, C ABI with "
                  "host buffers): K steps back to back, each uploading its x and mask "
                  "from pinned host memory and downloading its output to pinned host "
                  "memory on copy streams beside the neighbouring steps' forwards "
                  "(3 slots" + (", graph replay" if args.graph else "") + "); L2 not "
                  "flushed: every step streams its weights (far above L2) through it"}
    e2e_serial = {"value": tokens / (e2e_total * 1e-3 / K), "unit": "tokens/s",
                  "ms_per_step": e2e_total / K,
                  "how": "upload, eager forward and download one after another on "
                         "one stream, L2 flushed before each step"}
    return e2e, e2e_serial, e2e_ms


# --------------------------------------------------------- the CPU oracle

def oracle_sample(valid_idx, n: int):
    """n valid tokens spread evenly over the batch (all of them when n >= len)."""
    import numpy as np
    if n >= len(valid_idx):
        return valid_idx
    return valid_idx[np.unique(np.linspace(0, len(valid_idx) - 1, n).round().astype(np.int64))]


def oracle_pass(inp, tok, k: int):
    """The oracle's layer (routing from its own logits) on the given tokens: the
    timed unit of the CPU baseline.  Returns logits, ids, w and the float64
    accumulators of those tokens."""
    import oracle
    x = inp["x"][tok]
    v = inp["valid"][tok]
    logits = oracle.router_logits(x, v, inp["router_w"], inp["router_b"])
    ids, wt = oracle.topk(logits, v, k)
    oracle.route(ids, v, inp["workload"].E)
    sub = dict(inp)
    sub["x"] = x
    sub["valid"] = v
    acc = oracle.moe_tokens(sub, ids, wt)
    return logits, ids, wt, acc


def oracle_timed(inp, k: int, target_s: float):
    """Times the oracle on growing evenly spread samples of the valid tokens until
    one sample takes about target_s / 4 or more; returns the last sample's rate."""
    import numpy as np

    import oracle
    valid_idx = np.nonzero(inp["valid"].numpy())[0]
    cores = oracle.max_threads()          # the threads the oracle's loops actually use
    n = min(len(valid_idx), max(1, cores))
    while True:
        tok = oracle_sample(valid_idx, n)
        t0 = time.perf_counter()
        res = oracle_pass(inp, tok, k)
        dt = time.perf_counter() - t0
        if dt >= target_s / 4 or n >= len(valid_idx):
            return len(tok) / dt, tok, dt, cores, res
        n = min(len(valid_idx), int(n * max(2.0, target_s / max(dt, 1e-3))))


def parity_of_sample(inp, tok, res, gpu, k: int, fp8: bool) -> dict:
    """The GPU forward's rows of the sampled tokens against the oracle's:
    logits within 1e-4 (|l| + rms) elementwise; routing identical, or different
    only where the k-th and (k+1)-th logits lie within that tolerance; outputs
    max |gpu - oracle| / rms (oracle rms over the sample) on the tokens routed
    alike, against the layer's bound (2e-2 bf16, 6e-2 FP8)."""
    import numpy as np

    import oracle
    logits, ids, _, acc = res
    gl = gpu["logits"].numpy()[tok].astype(np.float64)
    ol = logits.astype(np.float64)
    rms_l = float(np.sqrt(np.mean(ol ** 2))) or 1.0
    logit_err = float(np.max(np.abs(gl - ol) / (np.abs(ol) + rms_l)))
    gids = gpu["topk_ids"].numpy()[tok]
    same = np.all(gids == ids, axis=1)
    mism = np.nonzero(~same)[0]
    near = 0
    for i in mism:
        # a near-tie: at every slot where the two differ, the chosen experts' oracle
        # logits lie within twice the 1e-4 logit tolerance of each other
        js = np.nonzero(gids[i] != ids[i])[0]
        gap = max(abs(ol[i][ids[i][j]] - ol[i][gids[i][j]]) for j in js)
        if gap <= 2e-4 * (np.abs(ol[i]).max() + rms_l):
            near += 1
    ref = oracle.bf16_to_f64(oracle.round_bf16(acc))
    out = oracle.bf16_to_f64(gpu["out"][tok])
    rms = float(np.sqrt(np.mean(acc ** 2))) or 1.0
    # against the exact (float64) layer output, as the parity tests measure it; and,
    # for information, against the oracle's own bf16 rounding of it (one bf16 ulp
    # of a large output element is itself 1-3 % of the rms)
    err = float(np.max(np.abs(out[same] - acc[same]))) / rms if same.any() else None
    err_r = float(np.max(np.abs(out[same] - ref[same]))) / rms if same.any() else None
    bound = 6e-2 if fp8 else 2e-2
    return {"tokens": int(len(tok)), "max_err_over_rms": err, "bound": bound,
            "within_bound": bool(err is not None and err <= bound),
            "max_err_vs_rounded_over_rms": err_r,
            "logit_rel_err_max": logit_err, "routing_mismatch_tokens": int(len(mism)),
            "routing_mismatch_near_tie": int(near),
            "how": "GPU forward of the timed batch vs the oracle on its own logits (float64 "
                   "accumulation before its final rounding), tokens spread evenly over the batch"}


def cpu_baseline(w, inp, gpu, target_s: float):
    """The oracle timed on the host cores on a bounded sample of the workload's
    valid tokens (about target_s of CPU work); when the GPU forward's outputs are
    given, the same oracle results give the sample's parity."""
    rate, tok, dt, cores, res = oracle_timed(inp, w.k, target_s)
    out = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": f"{len(tok)} valid tokens of {w.name} spread over the batch (all "
                     f"weights), {dt:.1f} s, double-precision C with OpenMP over tokens"}
    if gpu is not None:
        out["parity"] = parity_of_sample(inp, tok, res, gpu, w.k, w.wtype == "fp8")
    return out


def microbatch_rows(n_ranks: int, rows: int, lo: int, hi: int):
    """Rows of the gathered batch that one micro-batch holds: rows [lo, hi) of every
    rank's block of `rows`, in rank order (what the micro-batch's all_gather builds)."""
    return [r * rows + i for r in range(n_ranks) for i in range(lo, hi)]


def tp_reference_rows(d, w, rank: int, n_ranks: int, rows: int, ranges, dev):
    """This rank's rows [rank * rows, (rank + 1) * rows) as one GPU's plain forward
    computes them, before the layer is sharded: one forward per micro-batch, over the
    rows that micro-batch gathers from every rank (`ranges`: each micro-batch's
    [lo, hi) within a rank's rows), so that on one rank the layer must match it bit
    for bit (the router's split of its sums depends on the number of rows)."""
    import torch

    import mixture_experts_fp32_b200 as moe
    plan = moe.Plan(max_tokens=w.T, hidden=w.H, num_experts=w.E, top_k_max=w.k, inter=w.I,
                    num_shared=w.S, shared_inter=w.Is if w.S else 0, device=dev,
                    wtype=moe.MOE_W_BF16 if w.wtype == "bf16" else moe.MOE_W_FP8_E4M3_B128)
    wts = plan.weights(d["router_w"], d["router_b"], d["w_gate_up"], d["w_down"],
                       d.get("s_gate_up"), d.get("s_down"), d.get("ws_gate_up"),
                       d.get("ws_down"), d.get("ss_gate_up"), d.get("ss_down"))
    mine = torch.empty(rows, w.H, dtype=torch.bfloat16, device=dev)
    for lo, hi in ranges:
        idx = torch.tensor(microbatch_rows(n_ranks, rows, lo, hi), device=dev)
        out = torch.empty(len(idx), w.H, dtype=torch.bfloat16, device=dev)
        plan.forward(wts, d["x"][idx].contiguous(), d["valid"][idx].contiguous(), w.k, out)
        mine[lo:hi] = out[rank * (hi - lo):(rank + 1) * (hi - lo)]
    torch.cuda.synchronize()
    if plan.device_status() != 0:
        raise RuntimeError("device status set in the one-GPU reference forward")
    del plan, wts
    torch.cuda.empty_cache()
    return mine


def tp_check(out, ref, valid, n_ranks: int, fp8: bool) -> dict:
    """This rank's rows of the sharded layer against the one-GPU forward: identical
    bits on one rank; on several, max |diff| <= 2e-2 (bf16) / 6e-2 (FP8) x the rms of
    the reference's valid rows, and padding rows +0.0 exactly."""
    import torch
    pad = valid == 0
    pad_ok = bool(torch.all(out[pad].view(torch.int16) == 0).item()) if pad.any() else True
    if n_ranks == 1:
        same = bool(torch.equal(out.view(torch.int16), ref.view(torch.int16)))
        return {"ok": same and pad_ok, "rule": "bit-identical to the one-GPU forward",
                "identical": same, "padding_zero": pad_ok}
    v = valid != 0
    o, r = out[v].double(), ref[v].double()
    rms = float(r.pow(2).mean().sqrt()) if r.numel() else 1.0
    err = float((o - r).abs().max()) / (rms or 1.0) if r.numel() else 0.0
    bound = 6e-2 if fp8 else 2e-2
    return {"ok": err <= bound and pad_ok, "rule": f"max|diff| <= {bound} x rms",
            "max_err_over_rms": err, "padding_zero": pad_ok}


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
        w = workload_of(args, args.workload)
        if w.T % ws_n:
            raise SystemExit(f"{w.T} rows do not split over {ws_n} ranks")
        rows = w.T // ws_n
        inp = synth.make_inputs(w)        # the same seeded layer and gathered batch on every rank
        d = {key: (v.to(dev) if isinstance(v, torch.Tensor) else v) for key, v in inp.items()}
        del inp
        valid_tokens = int(d["valid"].sum().item())
        n_mb = args.tp_microbatches or (2 if w.wtype == "fp8" else 1)
        two = n_mb == 2 and rows >= 2
        # the reference for this rank's rows: one GPU's plain forward of what each
        # micro-batch gathers
        ref_rows = tp_reference_rows(d, w, rank, ws_n, rows,
                                     tp.split_rows(rows) if two else [(0, rows)], dev)
        pairs = args.tp_return == "pairs"
        kw = dict(E=w.E, H=w.H, I=w.I, S=w.S, Is=w.Is if w.S else 0, k_max=w.k,
                  fp8=w.wtype == "fp8", fused=args.tp_return != "nccl",
                  layout="ep" if pairs else args.tp_layout, pairs=pairs,
                  send_ctas=args.send_ctas)
        if two:
            layer = tp.TPMoETwoBatch(d, rows=rows, **kw)
        else:
            layer = tp.TPMoE(d, rows=rows, **kw)
        x_loc = d["x"][rank * rows:(rank + 1) * rows].contiguous()
        v_loc = d["valid"][rank * rows:(rank + 1) * rows].contiguous()
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
        plans = [h.plan for h in layer.halves] if hasattr(layer, "halves") else [layer.plan]
        if any(p.device_status() != 0 for p in plans):
            raise RuntimeError("device status set during warm-up")
        # every rank's own rows against the one-GPU forward, agreed on by all ranks
        # before anything is timed (bit for bit on one rank; on several the partial
        # sums are added in another order, so within the layer's tolerance)
        check = tp_check(out, ref_rows, v_loc, ws_n, w.wtype == "fp8")
        flag = torch.tensor([0.0 if check["ok"] else 1.0], device=dev)
        if ws_n > 1:
            dist.all_reduce(flag, op=dist.ReduceOp.MAX)
        if flag.item() != 0.0:
            raise RuntimeError(f"tensor-parallel rows differ from the one-GPU forward: {check}")
        K = args.steps
        # end to end through the layer's Python API: each step uploads this rank's rows
        # and mask from pinned host memory and downloads its output to pinned host memory
        x_host = x_loc.cpu().pin_memory()
        v_host = v_loc.cpu().pin_memory()
        o_host = torch.empty(rows, w.H, dtype=torch.bfloat16).pin_memory()
        x_dev, v_dev = torch.empty_like(x_loc), torch.empty_like(v_loc)
        e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(K)]
        dist.barrier()
        torch.cuda.synchronize()
        for e0, e1 in e2e_ev:
            e0.record()
            x_dev.copy_(x_host, non_blocking=True)
            v_dev.copy_(v_host, non_blocking=True)
            layer.forward(x_dev, v_dev, w.k, out)
            o_host.copy_(out, non_blocking=True)
            e1.record()
        torch.cuda.synchronize()
        dist.barrier()
        e2e_ms = reduce_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev) / K, "max", ws_n,
                                   dev)
        e2e_ok = bool(torch.equal(o_host.view(torch.int16), out.cpu().view(torch.int16)))
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
        if any(p.device_status() != 0 for p in plans):
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
                           "S": w.S, "parallelism": ("ep" if pairs else args.tp_layout)
                                                       + str(ws_n),
                           "partial_return": args.tp_return,
                           "send_ctas": args.send_ctas if pairs else None,
                           "micro_batches": 2 if hasattr(layer, "halves") else 1,
                           "l2": f"{L2_FLUSH_BYTES >> 20} MB written between timed steps"},
                "check": check,
                "e2e": {"value": valid_tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                        "ms_per_step": e2e_ms,
                        "h2d_bytes_per_step": ws_n * (x_host.numel() * 2 + v_host.numel()),
                        "d2h_bytes_per_step": ws_n * o_host.numel() * 2,
                        "output_matches_device": e2e_ok,
                        "how": "TP layer's forward with each rank's rows and mask uploaded "
                               "from pinned host memory and its output downloaded every "
                               "step (CUDA events, max over ranks, L2 not flushed)"},
                "gpu_launches": K * tp_launches_per_step(w, ws_n, rows, 2 if two else 1,
                                                         args.tp_return),
                "clocks": clk}))
    finally:
        del layer
        torch.cuda.synchronize()
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The reference arm: the CPU oracle (there is no installable reference
    implementation; the pages hold no code) on the host cores, rank 0 only.  Each
    step times the oracle on one bounded, evenly spread sample of the workload's
    valid tokens, sized so that the whole --steps/--warmup run ends within a few
    minutes; warm-up steps run a small sample."""
    import numpy as np

    import synth
    ws_n, rank, _ = dist_env()
    if rank != 0:
        return None
    w = workload_of(args, args.workload)
    inp = synth.make_inputs(w)
    valid_idx = np.nonzero(inp["valid"].numpy())[0]
    per_step = max(1.0, min(args.cpu_seconds, args.reference_seconds /
                            max(1, args.steps + args.warmup // 4 + 1)))
    rate, tok, dt, cores, _ = oracle_timed(inp, w.k, per_step)   # calibrates the sample
    small = oracle_sample(valid_idx, max(1, len(tok) // 8))
    for _ in range(max(args.warmup, 0)):
        oracle_pass(inp, small, w.k)
    rates, times = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_pass(inp, tok, w.k)
        dt = time.perf_counter() - t0
        times.append(dt)
        rates.append(len(tok) / dt)
    value = statistics.median(rates) if rates else 0.0
    res = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n,
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * statistics.median(times) if times else 0.0,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (Philox4x32-10, seed 0)", "impl": "reference",
           "config": {"workload": w.name, "T": w.T, "valid_tokens": int(len(valid_idx)),
                      "H": w.H, "E": w.E, "k": w.k, "I": w.I, "S": w.S, "Is": w.Is,
                      "wtype": w.wtype, "parallelism": "single GPU"},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                            "kind": "oracle",
                            "sample": f"{len(tok)} valid tokens of {w.name} per step, spread "
                                      f"over the batch (all weights); warm-up steps "
                                      f"{len(small)} tokens"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)
    return res


def workload_of(args, name: str):
    import synth
    w = synth.WORKLOADS[name]
    if args.experts:
        # a smaller copy of the workload (fewer experts) for profiler captures
        w = w.with_(name=f"{w.name}_e{args.experts}", E=args.experts, k=min(w.k, args.experts))
    return w


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None,
                    help="time this workload alone (default on one GPU: all timed workloads, "
                         "the Step3 decode step as the headline)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU work of the headline's CPU-baseline sample")
    ap.add_argument("--parity-seconds", type=float, default=4.0,
                    help="CPU work of the oracle sample of each other workload")
    ap.add_argument("--reference-seconds", type=float, default=150.0,
                    help="budget of the reference arm's timed steps together")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8-peak", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time eager forwards only (default: the headline is CUDA-graph replay)")
    ap.add_argument("--replicas", action="store_true",
                    help="under torchrun: N independent data-parallel replicas instead of "
                         "the tensor-parallel layer")
    ap.add_argument("--tp", action="store_true",
                    help="tensor-parallel layout over the N ranks (the default under torchrun; "
                         "with --tp alone the workload defaults to dp_padded)")
    ap.add_argument("--tp-return", default="fused", choices=["fused", "nccl", "pairs"],
                    help="fused: the combine stores each token's partial into its owner's "
                         "slab; nccl: reduce_scatter; pairs: expert-parallel per-pair return "
                         "from sender CTAs signalled by the down GEMM")
    ap.add_argument("--send-ctas", type=int, default=16,
                    help="with --tp-return pairs: CTAs of the down GEMM launch that send")
    ap.add_argument("--tp-layout", default="tp", choices=["tp", "ep"],
                    help="with --tp: split every expert's intermediate dimension (tp) or "
                         "the experts (ep) over the ranks")
    ap.add_argument("--tp-microbatches", type=int, default=0, choices=[0, 1, 2],
                    help="with --tp: micro-batches per step; 0 = one for the HBM-bound bf16 "
                         "decode batches (each micro-batch streams the rank's weights once), "
                         "two for the FP8 prefill")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the number of routed experts (profiling on a smaller case)")
    args = ap.parse_args(argv)
    ws_n = dist_env()[0]
    args.single = args.workload is not None or args.experts > 0
    if args.workload is None:
        args.workload = "dp_padded" if args.tp else DEFAULT_WORKLOAD
    if args.impl == "reference":
        run_reference(args)
    elif args.tp or (ws_n > 1 and not args.replicas):
        run_tp(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
