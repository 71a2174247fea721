"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: all logits and the complete routing (ids, weights, offsets,
permutation) against the oracle, outputs on rows the oracle computes one by one:
a spread sample, every padding row sampled, and one row of every 128-row tile of
the three heaviest routed groups and of the shared group (plus rows of small
groups), so that a tile-index or scheduling fault past the first waves shows.
The same rows' intermediates (permuted rows, h, y) are checked against float64
products of the GPU's own inputs, which locates a fault in one GEMM.  Routing is
also compared with the oracle's own logits: a token may route differently only
where its k-th and (k+1)-th logits lie within the 1e-4 logit tolerance."""
import gc

import numpy as np
import pytest
import torch

import oracle
import synth

from moe_harness import LOGIT_TOL, check_against_oracle, plan_for, rms, run_forward, to_device

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


def tile_rows(offsets: np.ndarray, E: int, S: int, valid: np.ndarray, heavy: int = 3,
              small: int = 4, stride: int = 128) -> np.ndarray:
    """Permuted row indices: the first row of every `stride`-row tile of the `heavy`
    largest routed groups and of the shared group (rows past offsets[E]), the last
    row of each such group, and the first row of `small` groups of 1..64 rows."""
    counts = np.diff(offsets)
    order = np.argsort(counts, kind="stable")[::-1]
    groups = [(offsets[e], offsets[e + 1]) for e in order[:heavy] if counts[e] > 0]
    nv = int(valid.sum())
    if S and nv:
        groups.append((offsets[-1], offsets[-1] + nv))            # the shared group
    rows = []
    for b, e in groups:
        rows += list(range(b, e, stride)) + [e - 1]
    tiny = [e for e in range(E) if 0 < counts[e] <= 64][:small]
    rows += [offsets[e] for e in tiny]
    return np.unique(np.asarray(rows, dtype=np.int64))


def routing_vs_own_logits(inp, res, k: int) -> dict:
    """Tokens whose top-k under the oracle's own logits differs from the GPU's,
    and whether each one is a near-tie at the k-th place."""
    valid = inp["valid"].numpy().astype(bool)
    ol = oracle.router_logits(inp["x"], inp["valid"], inp["router_w"], inp["router_b"])
    ids_o, _ = oracle.topk(ol, inp["valid"], k)
    ids_g = res["topk_ids"].numpy()
    diff = np.nonzero(np.any(ids_o != ids_g, axis=1) & valid)[0]
    r = rms(ol[valid])
    ties = 0
    for t in diff:
        # at every slot where the two differ, the experts chosen must have oracle logits
        # within twice the logit tolerance (a swap of near-equal logits)
        lt = ol[t].astype(np.float64)
        js = np.nonzero(ids_o[t] != ids_g[t])[0]
        gap = max(abs(lt[ids_o[t][j]] - lt[ids_g[t][j]]) for j in js)
        if gap <= 2 * LOGIT_TOL * (np.abs(lt).max() + r):
            ties += 1
    return {"mismatch": int(len(diff)), "near_tie": ties}


def dev_view(plan, ptr, shape, dtype):
    off = ptr - plan.workspace.data_ptr()
    nbytes = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
    return plan.workspace[off:off + nbytes].view(dtype).view(*shape).cpu()


def check_intermediates(inp, w, plan, res, rows: np.ndarray) -> dict:
    """x_perm, h and y of the given permuted rows against float64 products of the
    GPU's own inputs: h from the permuted row (gate/up GEMM + SwiGLU), y from the
    GPU's h row (down GEMM).  FP8: codes times their scales; h's tolerance is its
    quantisation step, y's the bf16 rounding."""
    v = plan.views()
    torch.cuda.synchronize()
    E = w.E
    group = dev_view(plan, v.group_offsets, (E + 1 + w.S,), torch.int32).numpy()
    R = int(group[-1])
    Rc = w.T * (w.k + w.S)
    rowtok = dev_view(plan, v.row_token, (R,), torch.int32).numpy()
    fp8 = w.wtype == "fp8"
    if fp8:      # the scale arrays, row-major [rows][groups]
        xsc = dev_view(plan, v.x_scale, (Rc, w.H // 128), torch.float32)
        hsc = dev_view(plan, v.h_scale, (Rc, v.h_stride // 128), torch.float32)
    worst = {"h": 0.0, "y": 0.0}
    for g in np.unique(np.searchsorted(group, rows, side="right") - 1):
        rs = rows[(rows >= group[g]) & (rows < group[g + 1])]
        routed = g < E
        I = w.I if routed else w.Is
        if fp8:
            def deq(codes, scales):
                c = codes.view(torch.float8_e4m3fn).double()
                return c * scales.double().repeat_interleave(128, 0).repeat_interleave(128, 1)
            Wgu = deq(inp["w_gate_up"][g] if routed else inp["ws_gate_up"],
                      inp["s_gate_up"][g] if routed else inp["ss_gate_up"])
            Wd = deq(inp["w_down"][g] if routed else inp["ws_down"],
                     inp["s_down"][g] if routed else inp["ss_down"])
        else:
            Wgu = (inp["w_gate_up"][g] if routed else inp["ws_gate_up"]).double()
            Wd = (inp["w_down"][g] if routed else inp["ws_down"]).double()
        for r in rs:
            r = int(r)
            if fp8:
                xc = dev_view(plan, v.x_perm + r * w.H, (w.H,), torch.uint8)
                xs = xsc[r].contiguous()
                xr = xc.view(torch.float8_e4m3fn).double() * xs.double().repeat_interleave(128)
                # the permuted row is the token's own quantisation
                q, s = oracle.quant_row_e4m3(
                    oracle.bf16_to_f64(inp["x"][rowtok[r]]).astype(np.float32))
                assert np.array_equal(xc.numpy(), q) and np.array_equal(xs.numpy(), s), r
                hc = dev_view(plan, v.h + r * v.h_stride, (I,), torch.uint8)
                hs = hsc[r, : I // 128].contiguous()
                hg = hc.view(torch.float8_e4m3fn).double() * hs.double().repeat_interleave(128)
                yg = dev_view(plan, v.y + 2 * r * w.H, (w.H,), torch.bfloat16).double()
            else:
                xr = dev_view(plan, v.x_perm + 2 * r * w.H, (w.H,), torch.bfloat16)
                assert torch.equal(xr, inp["x"][rowtok[r]]), r
                xr = xr.double()
                # two bf16 parts of h: rows 2r and 2r + 1
                h2 = dev_view(plan, v.h + 2 * 2 * r * v.h_stride, (2, v.h_stride), torch.bfloat16)
                hg = h2[0, :I].double() + h2[1, :I].double()
                yg = dev_view(plan, v.y + 4 * r * w.H, (w.H,), torch.float32).double()
            gg, uu = Wgu[:I] @ xr, Wgu[I:] @ xr
            href = torch.nn.functional.silu(gg) * uu
            if fp8:
                step = torch.maximum(href.abs() * 2.0 ** -4,
                                     hs.double().repeat_interleave(128) * 2.0 ** -10)
                herr = ((hg - href).abs() - step).max().item()
                assert herr <= 1e-4 * href.abs().max().item(), (g, r, herr)
                worst["h"] = max(worst["h"], herr / max(href.abs().max().item(), 1e-30))
            else:
                herr = (hg - href).abs().max().item()
                assert herr <= 2e-4 * href.abs().max().item() + 1e-6, (g, r, herr)
                worst["h"] = max(worst["h"], herr / max(href.abs().max().item(), 1e-30))
            yref = Wd @ hg
            yerr = (yg - yref).abs().max().item() / max(yref.abs().max().item(), 1e-30)
            assert yerr <= 1e-2, (g, r, yerr)
            worst["y"] = max(worst["y"], yerr)
    return worst


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w)
    d = to_device(inp)
    plan = plan_for(w)
    res = run_forward(plan, d, w.k)
    valid = inp["valid"].numpy()
    offsets = res["offsets"].numpy()
    # tiles of 128 rows (FP8 GEMMs, bf16 gate/up); the bf16 down GEMM's are 96
    prow = tile_rows(offsets, w.E, w.S, valid, stride=128 if w.wtype == "fp8" else 96)
    perm = res["perm"].numpy()
    # the tokens behind those permuted rows (shared rows: the valid tokens in order)
    vi = np.nonzero(valid)[0]
    toks = [perm[p] // w.k if p < offsets[-1] else vi[p - offsets[-1]] for p in prow]
    rows = np.unique(np.concatenate([sample_rows(valid), np.asarray(toks, dtype=np.int64)]))
    rep = check_against_oracle(inp, res, w.k, tokens=rows)
    inter = check_intermediates(inp, w, plan, res, prow)
    own = routing_vs_own_logits(inp, res, w.k)
    assert own["mismatch"] == own["near_tie"], own
    counts = np.diff(offsets)
    print(name, rep, inter, own, "rows checked", len(rows), "tiles", len(prow),
          "touched experts", int((counts > 0).sum()), "max rows/expert", int(counts.max()))
    del d, plan, res, inp
    gc.collect()
    torch.cuda.empty_cache()
