"""moe_route_from_logits_noalloc, the entry point for callers that cannot
allocate device memory (a framework pool that owns the device, a plain-C host
holding only device pointers, code running while its stream is captured): it
keeps its scratch in the library's static device array instead of a caller
workspace.  Its results must equal those of moe_route_from_logits, call after
call, while the array keeps the previous call's contents, and those of the CPU
oracle's top-k and routing on the same logits (crafted ties and padding rows
included), also above 1024 tokens, where the workspace path takes its
three-kernel route.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import mixture_experts_fp32_b200 as moe
import oracle

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
    # the oracle's own top-k and stable counting sort of the same logits
    ids_o, w_o = oracle.topk(lg.cpu(), vg.cpu(), k)
    _, off_o, perm_o, _ = oracle.route(ids_o, vg.cpu(), E)
    assert np.array_equal(ids_n.numpy(), ids_o)
    assert np.array_equal(off_n.numpy(), off_o)
    assert np.array_equal(perm_n[:npairs].numpy(), perm_o)
    assert np.abs(w_n.numpy().astype(np.float64) - w_o).max() <= WEIGHT_TOL


def test_noalloc_matches_workspace_routing_on_consecutive_calls():
    E, k = 48, 3
    plan = moe.Plan(max_tokens=600, hidden=128, num_experts=E, top_k_max=k, inter=128,
                    num_shared=1, shared_inter=128)
    _compare(plan, 600, E, k, seed=1)      # first call: also the per-device set-up
    _compare(plan, 77, E, k, seed=2)       # second call, smaller, over the first one's leftovers


def test_noalloc_above_one_chunk():
    # 3000 tokens: the workspace path runs its parallel count / scan / scatter
    # kernels, this entry point the one-block kernel over three 1024-token chunks
    E, k = 48, 3
    plan = moe.Plan(max_tokens=3000, hidden=128, num_experts=E, top_k_max=k, inter=128,
                    num_shared=1, shared_inter=128)
    _compare(plan, 3000, E, k, seed=6)
    _compare(plan, 2049, E, k, seed=7)


def _need(T, E, k, S):
    a = lambda n: (n + 255) // 256 * 256   # noqa: E731
    return 256 + a(4 * (E + 2)) + 2 * a(4 * T * (k + S))


def test_noalloc_deepseek_shape_and_size_limit():
    E, k, S = 256, 8, 1
    # the largest batch the 4 MiB array holds at this shape, and one token more
    t_max = max(T for T in range(58000, 58500) if _need(T, E, k, S) <= moe.MOE_STATIC_SCRATCH_BYTES)
    assert _need(t_max + 1, E, k, S) > moe.MOE_STATIC_SCRATCH_BYTES
    plan = moe.Plan(max_tokens=t_max + 1, hidden=128, num_experts=E, top_k_max=k, inter=128,
                    num_shared=S, shared_inter=128)
    _compare(plan, 1000, E, k, seed=3)
    _compare(plan, 999, E, k, seed=4)
    _compare(plan, t_max, E, k, seed=8)
    lg, vg = _logits(t_max + 1, E, 5)
    with pytest.raises(moe.MoeError) as ei:       # refused, nothing launched
        moe.moe_route_from_logits_noalloc(plan.handle, lg, vg, t_max + 1, k,
                                          *_outputs(t_max + 1, E, k))
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
