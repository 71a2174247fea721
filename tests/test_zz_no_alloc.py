"""moe_route_from_logits_noalloc, the entry point for callers that cannot
allocate device memory (a framework pool that owns the device, a plain-C host
holding only device pointers, code running while its stream is captured): it
keeps its scratch in the library's static device array instead of a caller
workspace.  Its results must equal those of moe_route_from_logits, call after
call, while the array keeps the previous call's contents.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import mixture_experts_fp32_b200 as moe

pytestmark = pytest.mark.gpu

WEIGHT_TOL = 2e-6   # the tolerance the routing weights are held to elsewhere


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_fp32_b200 import build
    build.build()
    moe.load()


def _logits(T, E, seed):
    rng = np.random.default_rng(seed)
    l = rng.standard_normal((T, E)).astype(np.float32)
    l[::4, : E // 3] = 0.25                   # exact ties: the lower expert index must win
    valid = (rng.random(T) > 0.15).astype(np.uint8)
    return torch.from_numpy(l).cuda(), torch.from_numpy(valid).cuda()


def _outputs(T, E, k):
    return (torch.full((T, k), -9, dtype=torch.int32, device="cuda"),
            torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda"),
            torch.full((T * k,), -9, dtype=torch.int32, device="cuda"),
            torch.full((E + 1,), -9, dtype=torch.int32, device="cuda"))


def _compare(plan, T, E, k, seed):
    lg, vg = _logits(T, E, seed)
    ref = _outputs(T, E, k)
    plan.route_from_logits(lg, vg, k, *ref)                       # caller workspace
    new = _outputs(T, E, k)
    moe.moe_route_from_logits_noalloc(plan.handle, lg, vg, T, k, *new)   # static scratch
    torch.cuda.synchronize()
    ids_r, w_r, perm_r, off_r = (t.cpu() for t in ref)
    ids_n, w_n, perm_n, off_n = (t.cpu() for t in new)
    npairs = int(off_r[-1])
    assert torch.equal(ids_n, ids_r)
    assert torch.equal(off_n, off_r)
    assert torch.equal(perm_n[:npairs], perm_r[:npairs])
    assert (w_n - w_r).abs().max().item() <= WEIGHT_TOL


def test_noalloc_matches_workspace_routing_on_consecutive_calls():
    E, k = 48, 3
    plan = moe.Plan(max_tokens=600, hidden=128, num_experts=E, top_k_max=k, inter=128,
                    num_shared=1, shared_inter=128)
    _compare(plan, 600, E, k, seed=1)      # first call: also the per-device set-up
    _compare(plan, 77, E, k, seed=2)       # second call, smaller, over the first one's leftovers


def test_noalloc_deepseek_shape_and_size_limit():
    E, k = 256, 8
    plan = moe.Plan(max_tokens=4096, hidden=128, num_experts=E, top_k_max=k, inter=128)
    _compare(plan, 1000, E, k, seed=3)
    _compare(plan, 999, E, k, seed=4)
    # 4096 tokens x 256 experts of logits alone fill the 4 MiB array: refused, nothing launched
    lg, vg = _logits(4096, E, 5)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_route_from_logits_noalloc(plan.handle, lg, vg, 4096, k, *_outputs(4096, E, k))
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
