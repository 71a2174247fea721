"""GPU parity of the whole forward pass against the CPU oracle, through the C
ABI, on small seeded shapes that span several tiles and ragged tails."""
import numpy as np
import pytest
import torch

import mixture_experts_fp32_b200 as moe
import oracle
import synth
from synth.workloads import Workload

from moe_harness import check_against_oracle, plan_for, run_forward, to_device

pytestmark = pytest.mark.gpu


def W(name, **kw):
    base = dict(T=16, H=256, E=8, k=2, I=128)
    base.update(kw)
    return Workload(name, **base)


CASES = [
    synth.WORKLOADS["tiny"],
    W("one_token", T=1),
    W("ragged_shared_is_ne_i", T=7, H=384, E=6, k=3, I=256, S=1, Is=384),
    W("e48_k3", T=33, H=512, E=48, k=3, I=256, router_sigma=0.2),
    W("e256_k8_bias", T=200, H=256, E=256, k=8, I=128, S=1, Is=128, bias="normal"),
    W("two_row_tiles", T=300, H=256, E=2, k=1, I=128),            # ~150 rows per expert
    W("skewed", T=300, H=256, E=4, k=2, I=256, bias="zipf", zipf_s=3.0),   # > 256 rows on one
    # a decode-sized batch whose Zipf load puts 46 and 62 rows on two of 16 experts
    W("decode_skewed", T=64, H=256, E=16, k=2, I=128, S=1, Is=128, bias="zipf", zipf_s=2.0),
    W("k_equals_e", T=9, H=256, E=4, k=4, I=128),
    W("padded", T=64, H=256, E=8, k=2, I=128, S=1, Is=128, mask="dp_padded",
      dp_rows=(3, 16, 0, 5)),
    W("wide", T=40, H=1024, E=16, k=2, I=640, S=1, Is=256, router_sigma=0.1),
]


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_fp32_b200 import build
    build.build()
    moe.load()


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_forward_matches_oracle(w):
    inp = synth.make_inputs(w)
    d = to_device(inp)
    plan = plan_for(w)
    res = run_forward(plan, d, w.k)
    rep = check_against_oracle(inp, res, w.k)
    print(w.name, rep)


def test_plan_larger_than_batch():
    w = W("small_in_big_plan", T=20, E=8, k=2)
    inp = synth.make_inputs(w)
    plan = plan_for(w, max_tokens=512)
    res = run_forward(plan, to_device(inp), 2)
    check_against_oracle(inp, res, 2)


def test_k_smaller_than_plan_max():
    w = W("k1_of_3", T=24, E=8, k=3, S=1, Is=128)
    inp = synth.make_inputs(w)
    plan = plan_for(w)
    res = run_forward(plan, to_device(inp), 1)
    check_against_oracle(inp, res, 1)


def test_padding_contents_do_not_matter():
    w = W("nan_padding", T=48, E=8, k=2, S=1, Is=128, mask="dp_padded", dp_rows=(5, 0, 12, 1))
    a = synth.make_inputs(w, masked_fill="normal")
    b = synth.make_inputs(w, masked_fill="nan")
    plan = plan_for(w)
    ra = run_forward(plan, to_device(a), 2)
    rb = run_forward(plan, to_device(b), 2)
    valid = a["valid"].numpy().astype(bool)
    assert torch.equal(ra["out"][valid].view(torch.int16), rb["out"][valid].view(torch.int16))
    assert (rb["out"][~valid].view(torch.int16) == 0).all()
    check_against_oracle(b, rb, 2)


def test_all_rows_padding():
    w = W("all_padding", T=32, S=1, Is=128, mask="dp_padded", dp_rows=(0, 0))
    inp = synth.make_inputs(w, masked_fill="nan")
    res = run_forward(plan_for(w), to_device(inp), 2)
    assert res["status"] == 0
    assert (res["out"].view(torch.int16) == 0).all()
    assert (res["offsets"] == 0).all()
    assert (res["topk_ids"] == -1).all()


def test_deterministic_bits():
    w = W("determinism", T=150, H=512, E=48, k=3, I=256, S=1, Is=256)
    d = to_device(synth.make_inputs(w))
    plan = plan_for(w)
    r1 = run_forward(plan, d, 3)
    r2 = run_forward(plan, d, 3)
    for key in ("out", "logits", "topk_ids", "topk_w", "perm", "offsets"):
        assert torch.equal(r1[key].view(torch.uint8), r2[key].view(torch.uint8)), key


def test_route_from_logits_bit_exact_with_ties():
    rng = np.random.default_rng(11)
    for T, E, k in ((16, 8, 2), (257, 48, 3), (1100, 256, 8), (5, 4, 4)):
        l = rng.standard_normal((T, E)).astype(np.float32)
        l[::3, : E // 2] = 0.5                          # many exact ties
        l[1::5] = np.round(l[1::5], 1)
        valid = (rng.random(T) > 0.2).astype(np.uint8)
        plan = moe.Plan(max_tokens=T, hidden=128, num_experts=E, top_k_max=k, inter=128)
        lg = torch.from_numpy(l).cuda()
        vg = torch.from_numpy(valid).cuda()
        ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
        wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
        perm = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        offs = torch.empty((E + 1,), dtype=torch.int32, device="cuda")
        plan.route_from_logits(lg, vg, k, ids, wts, perm, offs)
        torch.cuda.synchronize()
        ids_o, w_o = oracle.topk(l, valid, k)
        _, offs_o, perm_o, _ = oracle.route(ids_o, valid, E)
        assert np.array_equal(ids.cpu().numpy(), ids_o)
        assert np.array_equal(offs.cpu().numpy(), offs_o)
        assert np.array_equal(perm.cpu().numpy()[: offs_o[-1]], perm_o)
        assert np.abs(wts.cpu().numpy() - w_o).max() <= 2e-6
        assert plan.device_status() == 0


def test_wait_timeout_reports_and_recovers():
    """A wait limit of 0 makes the GEMMs' first unsatisfied wait give up: the
    kernels return early, the status bits say so, and the context stays usable."""
    w = W("timeout", T=64, H=512, E=8, k=2, I=256)
    inp = synth.make_inputs(w)
    d = to_device(inp)
    plan = plan_for(w)
    plan.set_wait_limit(0)
    res = run_forward(plan, d, 2)
    assert res["status"] & (moe.MOE_DEV_WAIT_TIMEOUT_GATE_UP | moe.MOE_DEV_WAIT_TIMEOUT_DOWN)
    assert plan.device_status() == 0                    # the read cleared it
    plan.set_wait_limit(2_000_000_000)
    res = run_forward(plan, d, 2)
    check_against_oracle(inp, res, 2)


def test_intermediate_rows_against_fp64():
    """The permuted rows, h = silu(g)*u and y of a few rows checked directly,
    so that a GEMM fault is located before the combine."""
    w = W("intermediates", T=40, H=384, E=5, k=2, I=256, S=1, Is=128, router_sigma=0.3)
    inp = synth.make_inputs(w)
    d = to_device(inp)
    plan = plan_for(w)
    res = run_forward(plan, d, 2)
    v = plan.views()
    torch.cuda.synchronize()
    R = int(res["offsets"][-1]) + w.T

    def dev_view(ptr, shape, dtype):
        """A slice of the workspace tensor at a device address from moe_get_workspace_views."""
        off = ptr - plan.workspace.data_ptr()
        nbytes = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
        return plan.workspace[off:off + nbytes].view(dtype).view(*shape).cpu()

    group = dev_view(v.group_offsets, (w.E + 2,), torch.int32).numpy()
    assert group[w.E] == int(res["offsets"][-1]) and group[w.E + 1] == R
    rowtok = dev_view(v.row_token, (R,), torch.int32).numpy()
    xp = dev_view(v.x_perm, (R, w.H), torch.bfloat16)
    h2 = dev_view(v.h, (2 * R, v.h_stride), torch.bfloat16)   # two parts a row
    h = h2[0::2].double() + h2[1::2].double()
    y = dev_view(v.y, (R, w.H), torch.float32)
    assert torch.equal(xp, inp["x"][torch.from_numpy(rowtok).long()])
    x64 = inp["x"].double()
    for r in list(range(0, R, 7)) + [R - 1]:
        g = int(np.searchsorted(group, r, side="right") - 1)
        if g < w.E:
            Wgu, Wd, I = inp["w_gate_up"][g].double(), inp["w_down"][g].double(), w.I
        else:
            Wgu, Wd, I = inp["ws_gate_up"].double(), inp["ws_down"].double(), w.Is
        xr = x64[rowtok[r]]
        gg, uu = Wgu[:I] @ xr, Wgu[I:] @ xr
        href = torch.nn.functional.silu(gg) * uu
        # hi = bf16(h), lo = bf16(h - hi): together about 16 significant bits
        hi = h2[2 * r, :I].double()
        assert torch.all((hi - href).abs()
                         <= 2.0 ** -8 * href.abs() + 1e-5 * href.abs().max()), (r, g)
        herr = (h[r, :I] - href).abs().max().item()
        assert herr <= 2e-4 * href.abs().max().item() + 1e-6, (r, g, herr)
        yref = Wd @ h[r, :I]
        yerr = (y[r].double() - yref).abs().max().item()
        assert yerr <= 1e-2 * yref.abs().max().item() + 1e-6, (r, g, yerr)


def test_router_split_made_once():
    """moe_split_router_weights writes Wr = W1 + W2 + W3 exactly (each part a bf16,
    the first the round-to-nearest bf16 of Wr, the later ones of the remainder,
    rows past E zero), and a forward that reads it equals, bit for bit, one that
    splits the router weights itself."""
    w = W("split_once", T=100, H=384, E=20, k=3, I=128, S=1, Is=128, router_sigma=0.3)
    inp = synth.make_inputs(w)
    d = to_device(inp)
    plan = plan_for(w)
    nbytes = moe.moe_router_split_bytes(plan.handle)
    E16 = (w.E + 15) // 16 * 16
    assert nbytes == 3 * E16 * w.H * 2
    split = torch.full((3, E16, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_split_router_weights(plan.handle, d["router_w"], split, nbytes)
    with pytest.raises(moe.MoeError):
        moe.moe_split_router_weights(plan.handle, d["router_w"], split, nbytes - 2)
    torch.cuda.synchronize()
    parts = split.cpu().double()
    wr = inp["router_w"].double()
    assert torch.equal(parts[:, : w.E].sum(0), wr)                    # exact, in fp64
    assert torch.equal(split[0, : w.E].cpu(), inp["router_w"].to(torch.bfloat16))
    assert torch.all(parts[:, w.E:] == 0)
    # each later part is at most half an ulp of bf16 of what came before it
    assert torch.all(parts[1].abs() <= parts[0].abs() * 2.0 ** -8)
    assert torch.all(parts[2].abs() <= parts[1].abs() * 2.0 ** -8)

    outs = []
    for wts in (plan.weights(d["router_w"], d["router_b"], d["w_gate_up"], d["w_down"],
                             ws_gate_up=d["ws_gate_up"], ws_down=d["ws_down"]),
                plan.weights(d["router_w"], d["router_b"], d["w_gate_up"], d["w_down"],
                             ws_gate_up=d["ws_gate_up"], ws_down=d["ws_down"],
                             split_router=False)):
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        plan.forward(wts, d["x"], d["valid"], w.k, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert wts.router_split is None
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert plan.device_status() == 0
