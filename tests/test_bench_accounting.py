"""The benchmark's roofline accounting against the step budgets worked out by hand for
each workload with every routed expert touched (bytes the layer must move: touched
experts' and the shared expert's weights, the router, valid input rows, all output rows;
flops of the expert FFNs and of the router)."""
import numpy as np
import pytest

import bench
import synth

# (workload, step GB, expert GFLOP, router GFLOP), all experts touched
BUDGETS = [
    ("step3_decode", 10.80, 225.5, 0.18),
    ("deepseek_decode", 22.65, 101.5, 0.47),
    ("dp_padded", 10.70, 750.4, 0.78),
    ("fp8_prefill", 11.56, 6494.0, 30.1),
]


@pytest.mark.parametrize("name,gb,gflop,router_gflop", BUDGETS)
def test_step_budget(name, gb, gflop, router_gflop):
    w = synth.WORKLOADS[name]
    valid = int(synth.workloads.valid_mask(w).sum())
    pairs = valid * w.k
    counts = np.full(w.E, pairs // w.E)
    counts[: pairs - counts.sum()] += 1              # every expert touched
    offsets = np.concatenate([[0], np.cumsum(counts)])
    a = bench.algorithmic(w, valid, offsets, w.k)
    assert a["touched_experts"] == w.E and a["routed_rows"] == pairs
    assert abs(a["step_bytes"] / 1e9 - gb) <= 0.006 * gb
    assert abs(a["expert_flops"] / 1e9 - gflop) <= 0.002 * gflop
    assert abs((a["step_flops"] - a["expert_flops"]) / 1e9 - router_gflop) <= 0.03 * router_gflop + 0.01
    # the gate/up kernel's share: two of the three expert matmuls
    assert abs(a["gate_up_flops"] / a["expert_flops"] - 2 / 3) < 1e-12


def test_untouched_experts_cost_no_weight_bytes():
    w = synth.WORKLOADS["step3_decode"]
    full = bench.algorithmic(w, w.T, np.arange(0, 49 * 16, 16), w.k)
    counts = np.zeros(w.E, dtype=int)
    counts[:10] = w.T * w.k // 10
    counts[0] += w.T * w.k - counts.sum()
    part = bench.algorithmic(w, w.T, np.concatenate([[0], np.cumsum(counts)]), w.k)
    per_expert = 3 * w.H * w.I * 2                   # gate, up and down, bf16
    assert part["touched_experts"] == 10
    assert full["step_bytes"] - part["step_bytes"] == (w.E - 10) * per_expert


def test_launch_count_per_step():
    # router, top-k; the permutation (1 kernel up to 1024 rows, 3 above); the gather or
    # FP8 quantisation; two GEMMs; the combine (the router weights' split is made once
    # with the weights, not per step)
    assert bench.launches_per_step(synth.WORKLOADS["step3_decode"]) == 7
    assert bench.launches_per_step(synth.WORKLOADS["fp8_prefill"]) == 9


def test_microbatch_rows_follow_the_all_gather():
    # two ranks of 4 rows, micro-batches [0, 2) and [2, 4): each gathers its slice of
    # every rank in rank order
    assert bench.microbatch_rows(2, 4, 0, 2) == [0, 1, 4, 5]
    assert bench.microbatch_rows(2, 4, 2, 4) == [2, 3, 6, 7]
    # together they cover the gathered batch once
    rows = sorted(bench.microbatch_rows(3, 5, 0, 2) + bench.microbatch_rows(3, 5, 2, 5))
    assert rows == list(range(15))
    # one micro-batch is the whole gathered batch in order
    assert bench.microbatch_rows(4, 3, 0, 3) == list(range(12))


def test_tp_launch_count_per_step():
    w = synth.WORKLOADS["step3_decode"]
    # one micro-batch: the layer over 8 x 32 gathered rows (7 kernels) + the owner's sum
    assert bench.tp_launches_per_step(w, 8, 32, 1, "fused") == 8
    # two micro-batches of 16 rows a rank
    assert bench.tp_launches_per_step(w, 8, 32, 2, "nccl") == 16
    # per-pair return: no combine, the pair sum, the shared expert as a one-expert layer
    assert bench.tp_launches_per_step(w, 8, 32, 1, "pairs") == 6 + 1 + 7
    # the FP8 prefill gathers 8192 rows: three route kernels and the quantisation
    assert bench.tp_launches_per_step(synth.WORKLOADS["fp8_prefill"], 8, 1024, 1, "fused") == 10


def test_step_spread():
    s = bench.step_spread([float(v) for v in range(1, 12)])     # 1..11 ms
    assert s == {"p10": 2.0, "p50": 6.0, "p90": 10.0}
    assert bench.step_spread([]) == {"p10": None, "p50": None, "p90": None}


def test_design_bytes():
    # x_perm, h and y of every routed and shared row, written once and read once
    w = synth.WORKLOADS["fp8_prefill"]
    pairs = w.T * w.k
    offsets = np.concatenate([[0], np.cumsum(np.full(w.E, pairs // w.E))])
    a = bench.algorithmic(w, w.T, offsets, w.k)
    R = pairs + w.T                                   # + the shared expert's rows
    per_row = (7168 + 56 * 4) + (2048 + 16 * 4) + 7168 * 2
    assert a["design_bytes"] == 2 * R * per_row       # about 3.5 GB
    w = synth.WORKLOADS["step3_decode"]
    a = bench.algorithmic(w, w.T, np.arange(0, 49 * 16, 16), w.k)
    assert a["design_bytes"] == 2 * (768 + 256) * (7168 * 2 + 5120 * 4 + 7168 * 4)


def test_expert_load_summary():
    offsets = np.array([0, 5, 5, 12, 12, 20])          # 4 experts: 5, 0, 7, 0, 8 -> E = 5
    e = bench.expert_load(offsets)
    assert e["touched"] == 3 and e["pairs"] == 20 and e["max_rows"] == 8
    assert e["min_rows_touched"] == 5 and abs(e["mean_rows_touched"] - 20 / 3) < 1e-12
    assert bench.expert_load(np.zeros(4, dtype=int)) == {"touched": 0}


def test_oracle_sample_spreads_over_the_batch():
    idx = np.arange(100, 200)
    s = bench.oracle_sample(idx, 5)
    assert list(s) == [100, 125, 150, 174, 199] or list(s) == [100, 125, 150, 175, 199]
    assert list(bench.oracle_sample(idx, 500)) == list(idx)


def test_tp_check_rules():
    import torch
    ref = torch.randn(6, 32).to(torch.bfloat16)
    valid = torch.tensor([1, 1, 1, 1, 0, 0], dtype=torch.uint8)
    ref[4:] = 0
    out = ref.clone()
    assert bench.tp_check(out, ref, valid, 1, False)["ok"]
    out[0, 0] = out[0, 0] + 0.5                        # any difference fails on one rank
    assert not bench.tp_check(out, ref, valid, 1, False)["ok"]
    r = bench.tp_check(out, ref, valid, 2, False)       # several ranks: the rms rule
    assert r["max_err_over_rms"] > 0 and r["ok"] == (r["max_err_over_rms"] <= 2e-2)
    small = ref.clone()
    small[1, 1] = (small[1, 1].float() * (1 + 2 ** -7)).to(torch.bfloat16)
    assert bench.tp_check(small, ref, valid, 2, False)["ok"]
    bad_pad = ref.clone()
    bad_pad[5, 3] = 1.0                                 # a padding row must stay +0.0
    assert not bench.tp_check(bad_pad, ref, valid, 2, False)["ok"]
