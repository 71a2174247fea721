"""The seeded generator (Philox4x32-10 known answers, determinism) and the
workload definitions against the figures the pages print."""
import json
import os

import numpy as np
import torch

import synth
from synth.workloads import WORKLOADS, make_inputs, valid_mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def test_philox_known_answers():
    # Known-answer vectors published with the Random123 library (Salmon et al., SC'11).
    assert synth.philox4x32_10([0, 0, 0, 0], [0, 0]) == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C,
                                                         0x9B00DBD8]
    assert synth.philox4x32_10([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2) == [
        0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]
    assert synth.philox4x32_10([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344],
                               [0xA4093822, 0x299F31D0]) == [0xD16CFE09, 0x94FDCCEB, 0x5001E420,
                                                             0x24126EA1]


def test_normals_are_chunk_invariant_and_standard():
    a = synth.normal_f32(0, 1, 1 << 20)
    b = synth.normal_f32(0, 1, 999, start=4097)
    assert np.array_equal(a[4097:4097 + 999], b)
    assert abs(a.mean()) < 5e-3 and abs(a.std() - 1) < 5e-3
    c = synth.normal_f32(0, 2, 1 << 10)
    assert not np.array_equal(a[:1 << 10], c)
    u = synth.uniform_f64(0, 3, 1 << 16)
    assert u.min() > 0 and u.max() < 1 and abs(u.mean() - 0.5) < 5e-3


def test_bf16_tensor_is_torch_rounding_of_fp32_draws():
    t = synth.normal_bf16(0, 9, (7, 33), 0.5)
    ref = torch.from_numpy(synth.normal_f32(0, 9, 7 * 33, 0.5)).to(torch.bfloat16).view(7, 33)
    assert torch.equal(t, ref)


def test_page_facts_pin_the_workloads():
    facts = json.load(open(GOLDEN))
    s3 = WORKLOADS["step3_decode"]
    f = facts["step3_expert_selection"]
    assert (s3.E, s3.k) == (f["experts"], f["top_k"])

    f = facts["dp_attention_padding"]
    dp = WORKLOADS["dp_padded"]
    m = valid_mask(dp)
    assert dp.T == f["ranks"] * f["prefill_rank_tokens"]
    per = dp.T // f["ranks"]
    rows = [int(m[r * per:(r + 1) * per].sum()) for r in range(f["ranks"])]
    assert sorted(rows) == [f["decode_rank_tokens"]] * 7 + [f["prefill_rank_tokens"]]
    waste = 1.0 - m.sum() / dp.T
    assert round(100 * waste) == f["padding_waste_percent"]

    f = facts["microbatch_split"]
    assert sum(f["requests"]) == f["total_tokens"]
    assert f["boundary_split"] == [f["requests"][0], sum(f["requests"][1:])]
    assert round(f["boundary_split"][1] / f["boundary_split"][0], 2) == f["boundary_ratio"]
    assert f["even_split"] == [f["total_tokens"] // 2] * 2
    assert WORKLOADS["fp8_prefill"].T == f["even_split"][0]


def test_make_inputs_shapes_and_nan_padding():
    w = WORKLOADS["tiny"].with_(mask="dp_padded", dp_rows=(2, 1, 4, 0))
    a = make_inputs(w, masked_fill="nan")
    assert a["x"].shape == (16, 256) and a["w_gate_up"].shape == (8, 256, 256)
    assert a["w_down"].shape == (8, 256, 128)
    valid = a["valid"].numpy().astype(bool)
    assert torch.isnan(a["x"][torch.from_numpy(~valid)]).all()
    assert not torch.isnan(a["x"][torch.from_numpy(valid)]).any()
    z = WORKLOADS["fp8_prefill"].with_(T=4, H=256, E=3, I=128, Is=128)
    b = make_inputs(z)
    assert b["w_gate_up"].dtype == torch.uint8 and b["s_gate_up"].shape == (3, 2, 2)
    assert b["router_b"].shape == (3,)
