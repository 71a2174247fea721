"""GPU parity of the FP8 block-scale path (e4m3 weights with 128x128 fp32
scales, activations quantised 1x128 inside the forward) against the oracle,
which quantises exactly as the pages' block-scale reading says."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.workloads import Workload

from moe_harness import check_against_oracle, plan_for, run_forward, to_device

pytestmark = pytest.mark.gpu


def W(name, **kw):
    base = dict(T=16, H=256, E=8, k=2, I=128, wtype="fp8", w_sigma=0.05)
    base.update(kw)
    return Workload(name, **base)


CASES = [
    W("fp8_tiny", router_sigma=0.02),
    W("fp8_one_token", T=1),
    W("fp8_shared_is_ne_i", T=40, H=512, E=16, k=4, I=256, S=1, Is=384, router_sigma=0.1),
    W("fp8_zipf_many_rows", T=300, H=256, E=32, k=8, I=128, S=1, Is=128, bias="zipf"),
    W("fp8_padded", T=64, H=384, E=8, k=2, I=256, S=1, Is=128, mask="dp_padded",
      dp_rows=(3, 16, 0, 5)),
]


@pytest.fixture(scope="module", autouse=True)
def built():
    import mixture_experts_fp32_b200 as moe
    from mixture_experts_fp32_b200 import build
    build.build()
    moe.load()


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_fp8_forward_matches_oracle(w):
    inp = synth.make_inputs(w)
    plan = plan_for(w)
    res = run_forward(plan, to_device(inp), w.k)
    rep = check_against_oracle(inp, res, w.k)
    print(w.name, rep)


def test_fp8_activation_codes_bit_exact():
    """The permuted e4m3 rows and their scales equal the oracle's quantisation
    of the same rows, code for code (both divide in fp32, round to nearest even
    and saturate)."""
    w = W("fp8_codes", T=37, H=640, E=6, k=3, I=128, S=1, Is=256, router_sigma=0.2)
    inp = synth.make_inputs(w)
    plan = plan_for(w)
    res = run_forward(plan, to_device(inp), w.k)
    v = plan.views()
    torch.cuda.synchronize()
    R = int(res["offsets"][-1]) + w.T

    def dev_view(ptr, n, dtype):
        off = ptr - plan.workspace.data_ptr()
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        return plan.workspace[off:off + nbytes].view(dtype).cpu()

    rowtok = dev_view(v.row_token, R, torch.int32).numpy()
    codes = dev_view(v.x_perm, R * w.H, torch.uint8).numpy().reshape(R, w.H)
    scales = dev_view(v.x_scale, R * (w.H // 128), torch.float32).numpy().reshape(R, w.H // 128)
    xf = oracle.bf16_to_f64(inp["x"]).reshape(w.T, w.H).astype(np.float32)
    for r in range(R):
        q, s = oracle.quant_row_e4m3(xf[rowtok[r]])
        assert np.array_equal(codes[r], q), r
        assert np.array_equal(scales[r], s), r
