"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: all logits and the complete routing (ids, weights, offsets,
permutation) against the oracle, outputs on a sample of rows the oracle
computes one by one (plus every padding row)."""
import gc

import numpy as np
import pytest
import torch

import synth

from moe_harness import check_against_oracle, plan_for, run_forward, to_device

pytestmark = pytest.mark.gpu

FULL = ["step3_decode", "deepseek_decode", "dp_padded", "fp8_prefill"]


def sample_rows(valid: np.ndarray, n_random: int = 6, seed: int = 0) -> np.ndarray:
    vi = np.nonzero(valid)[0]
    pi = np.nonzero(valid == 0)[0]
    rng = np.random.default_rng(seed)
    picks = list(vi[:3]) + list(vi[-2:]) + list(rng.choice(vi, min(n_random, len(vi)),
                                                           replace=False))
    if len(pi):
        picks += list(pi[:2]) + list(rng.choice(pi, min(2, len(pi)), replace=False))
    return np.unique(np.asarray(picks, dtype=np.int64))


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w)
    d = to_device(inp)
    plan = plan_for(w)
    res = run_forward(plan, d, w.k)
    rows = sample_rows(inp["valid"].numpy())
    rep = check_against_oracle(inp, res, w.k, tokens=rows)
    counts = np.diff(res["offsets"].numpy())
    print(name, rep, "touched experts", int((counts > 0).sum()), "max rows/expert",
          int(counts.max()))
    del d, plan, res, inp
    gc.collect()
    torch.cuda.empty_cache()
