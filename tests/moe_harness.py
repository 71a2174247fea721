"""Shared test helpers: run the CUDA library through its C ABI on seeded inputs
and compare with the CPU oracle.  Tolerances (all over valid rows):

  logits   |gpu - oracle| <= 1e-4 * (|oracle| + rms(oracle))          (fp32 sums vs fp64)
  routing  ids, perm, offsets identical to the oracle's routing of the GPU's logits
  weights  |gpu - oracle| <= 2e-6                                       (expf vs exp in fp64)
  output   max |gpu - oracle| <= 2e-2 * rms(oracle)  (bf16 weights)
           max |gpu - oracle| <= 6e-2 * rms(oracle)  (e4m3 block-scaled weights)
  padding  rows with valid = 0 are exactly +0.0
"""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_fp32_b200 as moe
import oracle

OUT_TOL = {"bf16": 2e-2, "fp8": 6e-2}
LOGIT_TOL = 1e-4
WEIGHT_TOL = 2e-6


def plan_for(w, max_tokens=None):
    return moe.Plan(max_tokens=max_tokens or w.T, hidden=w.H, num_experts=w.E, top_k_max=w.k,
                    inter=w.I, num_shared=w.S, shared_inter=w.Is if w.S else 0,
                    wtype=moe.MOE_W_BF16 if w.wtype == "bf16" else moe.MOE_W_FP8_E4M3_B128)


def to_device(inp: dict, device="cuda") -> dict:
    d = {}
    for key, v in inp.items():
        d[key] = v.to(device) if isinstance(v, torch.Tensor) else v
    return d


def weights_of(d: dict) -> moe.moe_weights:
    return moe.make_weights(d["router_w"], d.get("router_b"), d["w_gate_up"], d["w_down"],
                            d.get("s_gate_up"), d.get("s_down"), d.get("ws_gate_up"),
                            d.get("ws_down"), d.get("ss_gate_up"), d.get("ss_down"))


def run_forward(plan: moe.Plan, d: dict, k: int, valid_arg=True):
    """One forward through moe_forward with every debug output requested."""
    w = d["workload"]
    T = d["x"].shape[0]
    dev = d["x"].device
    out = torch.full((T, w.H), float("nan"), dtype=torch.bfloat16, device=dev)
    dbg_t = {
        "logits": torch.full((T, w.E), float("nan"), dtype=torch.float32, device=dev),
        "topk_ids": torch.full((T, k), -7, dtype=torch.int32, device=dev),
        "topk_w": torch.full((T, k), float("nan"), dtype=torch.float32, device=dev),
        "perm": torch.full((max(T * k, 1),), -7, dtype=torch.int32, device=dev),
        "offsets": torch.full((w.E + 1,), -7, dtype=torch.int32, device=dev),
    }
    dbg = moe.make_debug(**dbg_t)
    plan.forward(weights_of(d), d["x"], d["valid"] if valid_arg else None, k, out, dbg=dbg)
    torch.cuda.synchronize()
    status = plan.device_status()
    res = {key: v.cpu() for key, v in dbg_t.items()}
    res["out"] = out.cpu()
    res["status"] = status
    return res


def rms(a: np.ndarray) -> float:
    return float(np.sqrt(np.mean(np.square(a)))) if a.size else 0.0


def check_against_oracle(inp: dict, res: dict, k: int, tokens=None, check_routing=True):
    """Asserts every stated tolerance; returns a dict of measured errors."""
    w = inp["workload"]
    valid = inp["valid"].numpy().astype(bool)
    T = valid.size
    assert res["status"] == 0, f"device status bits {res['status']:#x}"

    # a1: logits
    gl = res["logits"].numpy()
    ol = oracle.router_logits(inp["x"], inp["valid"], inp["router_w"], inp["router_b"])
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    vt = tok[valid[tok]]
    lerr = np.abs(gl[vt] - ol[vt])
    lbound = LOGIT_TOL * (np.abs(ol[vt]) + rms(ol[vt]))
    assert np.all(lerr <= lbound), f"logit error {float((lerr / np.maximum(lbound, 1e-30)).max())}x"
    assert np.all(gl[~valid] == 0)

    # a2, a3: routing, bit-exact from the GPU's own logits
    ids_o, w_o = oracle.topk(gl, inp["valid"], k)
    counts, offs, perm, inv = oracle.route(ids_o, inp["valid"], w.E)
    ids_g = res["topk_ids"].numpy()
    report = {"logit_err_max_rel": float((lerr / np.maximum(lbound / LOGIT_TOL, 1e-30)).max())
              if lerr.size else 0.0}
    if check_routing:
        assert np.array_equal(ids_g, ids_o), "top-k ids differ"
        assert np.array_equal(res["offsets"].numpy(), offs), "expert offsets differ"
        npairs = int(offs[-1])
        assert np.array_equal(res["perm"].numpy()[:npairs], perm), "permutation differs"
        werr = np.abs(res["topk_w"].numpy() - w_o)
        assert np.all(werr[valid] <= WEIGHT_TOL), f"routing weight error {werr[valid].max()}"
        assert np.all(res["topk_w"].numpy()[~valid] == 0)
        report["weight_err_max"] = float(werr[valid].max()) if valid.any() else 0.0

    # a4-a6: outputs, oracle driven by the same routing
    acc = oracle.moe_tokens(inp, ids_o, w_o, tok)
    ref = oracle.bf16_to_f64(oracle.round_bf16(acc)).reshape(len(tok), w.H)
    got = res["out"][torch.from_numpy(tok)].double().numpy()
    vm = valid[tok]
    scale = rms(acc[vm])
    err = np.abs(got[vm] - acc[vm])
    tol = OUT_TOL[w.wtype] * scale
    report.update(out_rms=scale, out_err_max=float(err.max()) if err.size else 0.0,
                  out_err_rel=float(err.max() / scale) if err.size and scale > 0 else 0.0,
                  out_err_vs_rounded=float(np.abs(got[vm] - ref[vm]).max()) if err.size else 0.0)
    assert np.all(err <= tol), f"output error {report['out_err_rel']:.4g} x rms > {OUT_TOL[w.wtype]}"
    pad = res["out"][torch.from_numpy(tok[~vm])]
    assert torch.equal(pad.view(torch.int16), torch.zeros_like(pad.view(torch.int16))), \
        "padding rows are not +0.0"
    return report
