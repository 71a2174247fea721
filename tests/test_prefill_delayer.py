"""The prefill admission policy against the page's padding example (one rank prefilling
1024 tokens while seven decode 16 pads the gathered batch to 86 % padding), against its
rules (all together, timeout, low-water mark), on simulated traffic, and across four gloo
ranks that must reach the same decision from the gathered states."""
import json
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from mixture_experts_fp32_b200 import prefill_delayer as pd

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def page_states(waited=0):
    f = json.load(open(GOLDEN))["dp_attention_padding"]
    states = [pd.RankState(0, f["decode_rank_tokens"], 0) for _ in range(f["ranks"])]
    states[4] = pd.RankState(f["prefill_rank_tokens"], f["decode_rank_tokens"], waited)
    return f, states


def test_page_example_immediate_policy_pads_86_percent():
    f, states = page_states()
    go = pd.decide(states, pd.Policy.immediate())
    assert go == [False] * 4 + [True] + [False] * 3
    rows = pd.rows_this_step(states, go)
    assert rows == [16] * 4 + [1024] + [16] * 3
    assert round(100 * pd.padding_waste(rows)) == f["padding_waste_percent"]
    assert abs(pd.padding_waste(rows) - (1 - 1136 / 8192)) < 1e-12


def test_page_example_delayer_holds_the_lone_prefill():
    _, states = page_states(waited=0)
    go = pd.decide(states, pd.Policy(timeout_steps=8))
    assert not any(go)
    assert pd.padding_waste(pd.rows_this_step(states, go)) == 0.0   # all decode 16
    # at the timeout it goes through
    _, states = page_states(waited=8)
    assert pd.decide(states, pd.Policy(timeout_steps=8))[4]


def test_rules():
    P = pd.Policy(timeout_steps=5, low_water=2)
    s = lambda p, d, w=0: pd.RankState(p, d, w)
    assert pd.decide([s(0, 9), s(0, 9)], P) == [False, False]            # nothing ready
    assert pd.decide([s(100, 9), s(200, 9)], P) == [True, True]          # all together
    assert pd.decide([s(100, 9), s(0, 9)], P) == [False, False]          # held
    assert pd.decide([s(100, 9, 5), s(0, 9)], P) == [True, False]        # timeout
    assert pd.decide([s(100, 2), s(0, 9)], P) == [True, False]           # low-water mark
    # a forced rank takes every ready rank with it
    assert pd.decide([s(100, 9, 5), s(50, 9, 0), s(0, 9)], P) == [True, True, False]


def test_zero_timeout_is_the_immediate_policy():
    rng = np.random.default_rng(3)
    for _ in range(500):
        G = int(rng.integers(1, 9))
        states = [pd.RankState(int(rng.integers(0, 2)) * int(rng.integers(1, 2000)),
                               int(rng.integers(0, 40)), int(rng.integers(0, 10)))
                  for _ in range(G)]
        go = pd.decide(states, pd.Policy(timeout_steps=0, low_water=0))
        assert go == [st.prefill_tokens > 0 for st in states]


def test_simulation_invariants():
    tr = pd.Traffic(steps=1500, seed=1)
    imm = pd.simulate(tr, pd.Policy.immediate())
    assert imm.max_held == 0
    # the page's regime: about 86 % of a gathered batch is padding when one rank prefills
    assert 0.8 < imm.prefill_step_waste < 0.9
    for timeout in (4, 16, 64):
        dly = pd.simulate(tr, pd.Policy(timeout_steps=timeout))
        assert dly.max_held <= timeout                     # the timeout bounds the hold
        assert dly.mean_waste < imm.mean_waste             # and the padding drops
        assert dly.gathered_rows >= dly.real_rows
    slow = pd.simulate(tr, pd.Policy(timeout_steps=64))
    fast = pd.simulate(tr, pd.Policy(timeout_steps=4))
    assert slow.mean_waste < fast.mean_waste               # longer holds, less padding
    assert slow.mean_delay > fast.mean_delay               # at the cost of admission delay


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        rng = np.random.default_rng(11)             # the same draws on every rank
        out = []
        for _ in range(40):
            states = [pd.RankState(int(rng.integers(0, 2)) * int(rng.integers(1, 2000)),
                                   int(rng.integers(0, 20)), int(rng.integers(0, 12)))
                      for _ in range(world)]
            policy = pd.Policy(timeout_steps=int(rng.integers(0, 10)),
                               low_water=int(rng.integers(0, 4)))
            mine = pd.decide_distributed(states[rank], policy)
            every = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
            dist.all_gather(every, torch.tensor([int(mine)]))
            out.append(([bool(e.item()) for e in every], pd.decide(states, policy)))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_four_gloo_ranks_agree_on_the_decision():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 4, port, q)) for r in range(4)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for _ in range(4):
        rank, out = q.get(timeout=10)
        for gathered, expected in out:
            assert gathered == expected
