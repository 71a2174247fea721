"""Prefill admission for data-parallel ranks that feed one all_gather-padded MoE layer.

With DP attention in front of a tensor-parallel MoE, every step all_gathers the hidden
rows of all ranks, and the gather pads each rank to the largest rank's row count.  One
rank in prefill (~1024 tokens) while the other seven decode (~16 tokens each) pads the
gathered batch to 8 x 1024 rows of which 1136 are real: 86 % padding.  The remedy the
page describes is a scheduling one: a rank whose prefill is ready is not switched to
prefill at once; the ranks' states are observed together and the ranks enter prefill
together, or a timeout / low-water-mark rule lets the waiting prefill through (DP
Attention and TBO for DeepSeek-V4 on MI355X, §もう一つの柱：PrefillDelayer).

Readings (the page gives the rule's parts, not its parameters):
  * all together: when every rank has a prefill ready, all of them run it this step;
  * timeout: a prefill held back for `timeout_steps` steps is let through;
  * low-water mark: a rank whose running decode batch has fallen to `low_water`
    requests or fewer is let through (holding it back would leave it nearly idle);
  * when any rank is let through, every rank with a ready prefill goes with it: the
    gather is padded to the prefill length that step anyway, so joining costs nothing.
`timeout_steps = 0` is the immediate policy (every ready prefill runs at once).

The decision is a pure function of all ranks' states, so every rank computes the same
decision from the same all_gathered state vector (`decide_distributed`).  `simulate`
runs seeded arrival / decode traffic on G ranks through a policy and reports the padding
of the gathered MoE batches and the admission delay.  Host logic only.
"""
from __future__ import annotations

import json
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np


@dataclass(frozen=True)
class RankState:
    prefill_tokens: int     # tokens of the prefill ready on this rank (0: none)
    decode_requests: int    # running decode requests (one token each per decode step)
    waited: int             # steps the ready prefill has been held back


@dataclass(frozen=True)
class Policy:
    timeout_steps: int = 8
    low_water: int = 0

    @staticmethod
    def immediate() -> "Policy":
        return Policy(timeout_steps=0, low_water=0)


def decide(states: Sequence[RankState], policy: Policy) -> List[bool]:
    """Which ranks run their ready prefill this step (the same answer on every rank)."""
    ready = [s.prefill_tokens > 0 for s in states]
    if not any(ready):
        return [False] * len(states)
    forced = any(r and (s.waited >= policy.timeout_steps or s.decode_requests <= policy.low_water)
                 for r, s in zip(ready, states))
    if all(ready) or forced:
        return ready
    return [False] * len(states)


def rows_this_step(states: Sequence[RankState], prefill: Sequence[bool]) -> List[int]:
    """Real rows each rank contributes to the gathered MoE batch."""
    return [s.prefill_tokens if p else s.decode_requests for s, p in zip(states, prefill)]


def padding_waste(rows: Sequence[int]) -> float:
    """Fraction of the padded gather (G ranks x the largest rank's rows) that is padding."""
    m = max(rows)
    return 0.0 if m == 0 else 1.0 - sum(rows) / (len(rows) * m)


def decide_distributed(local: RankState, policy: Policy, group=None) -> bool:
    """Gathers every rank's state (3 integers) and returns this rank's decision; all
    ranks evaluate `decide` on the same gathered vector, so they agree."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    mine = torch.tensor([local.prefill_tokens, local.decode_requests, local.waited],
                        dtype=torch.int64)
    allv = [torch.zeros(3, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(allv, mine, group=group)
    states = [RankState(int(v[0]), int(v[1]), int(v[2])) for v in allv]
    return decide(states, policy)[dist.get_rank(group)]


# ---------------------------------------------------------------------- simulation

@dataclass
class Traffic:
    """Seeded per-rank traffic: prefill requests arrive on each rank as a Bernoulli
    process per step; a request's prompt and output lengths are drawn uniformly
    around the given means; a rank admits one prefill per step."""
    ranks: int = 8
    steps: int = 4000
    arrival_prob: float = 0.02          # per rank per step
    prompt_mean: int = 1024
    prompt_spread: float = 0.25         # uniform in mean * (1 +- spread)
    output_mean: int = 256
    output_spread: float = 0.5
    initial_decode: int = 16            # running requests per rank at step 0
    seed: int = 0


@dataclass
class SimResult:
    steps: int
    mean_waste: float                   # padding fraction of all gathered rows
    prefill_step_waste: float           # the same over steps that ran some prefill
    gathered_rows: int
    real_rows: int
    prefills: int
    mean_delay: float                   # steps from arrival to admission (queueing included)
    max_delay: int
    max_held: int                       # steps a ready prefill at the head was held back
    decode_tokens: int
    waste_hist: List[float] = field(default_factory=list)

    def as_dict(self):
        d = dict(self.__dict__)
        d.pop("waste_hist")
        return d


def simulate(traffic: Traffic, policy: Policy) -> SimResult:
    rng = np.random.default_rng(traffic.seed)
    G = traffic.ranks
    # per rank: queue of (prompt, output) ready to prefill, with the step they became ready
    queue: List[List[tuple]] = [[] for _ in range(G)]
    # per rank: remaining output tokens of each running request
    running: List[List[int]] = []
    for _ in range(G):
        running.append(list(rng.integers(1, 2 * traffic.output_mean,
                                         size=traffic.initial_decode)))
    waited = [0] * G
    gathered = real = prefills = decode_tokens = 0
    delays: List[int] = []
    held: List[int] = []
    wastes: List[float] = []
    pre_gathered = pre_real = 0

    def draw(mean, spread):
        lo, hi = mean * (1 - spread), mean * (1 + spread)
        return max(1, int(round(rng.uniform(lo, hi))))

    for step in range(traffic.steps):
        for r in range(G):
            if rng.random() < traffic.arrival_prob:
                queue[r].append((draw(traffic.prompt_mean, traffic.prompt_spread),
                                 draw(traffic.output_mean, traffic.output_spread), step))
        states = [RankState(queue[r][0][0] if queue[r] else 0, len(running[r]),
                            waited[r] if queue[r] else 0) for r in range(G)]
        go = decide(states, policy)
        rows = rows_this_step(states, go)
        m = max(rows)
        if m == 0:
            continue
        gathered += G * m
        real += sum(rows)
        wastes.append(padding_waste(rows))
        if any(go):
            pre_gathered += G * m
            pre_real += sum(rows)
        for r in range(G):
            if go[r]:
                prompt, out, ready_at = queue[r].pop(0)
                delays.append(step - ready_at)
                held.append(states[r].waited)
                prefills += 1
                running[r].append(out)
                waited[r] = 0
            else:
                decode_tokens += len(running[r])
                running[r] = [t - 1 for t in running[r] if t > 1]
                if queue[r]:
                    waited[r] += 1
    return SimResult(
        steps=traffic.steps,
        mean_waste=1.0 - real / gathered if gathered else 0.0,
        prefill_step_waste=1.0 - pre_real / pre_gathered if pre_gathered else 0.0,
        gathered_rows=gathered, real_rows=real, prefills=prefills,
        mean_delay=float(np.mean(delays)) if delays else 0.0,
        max_delay=int(max(delays)) if delays else 0,
        max_held=int(max(held)) if held else 0,
        decode_tokens=decode_tokens, waste_hist=wastes)


def main(argv: Optional[Sequence[str]] = None) -> None:
    import argparse
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--ranks", type=int, default=8)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--arrival-prob", type=float, default=0.02)
    ap.add_argument("--timeout", type=int, default=64)
    ap.add_argument("--low-water", type=int, default=0)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args(argv)
    tr = Traffic(ranks=a.ranks, steps=a.steps, arrival_prob=a.arrival_prob, seed=a.seed)
    imm = simulate(tr, Policy.immediate())
    dly = simulate(tr, Policy(timeout_steps=a.timeout, low_water=a.low_water))
    print(json.dumps({"traffic": tr.__dict__, "immediate": imm.as_dict(),
                      "delayer": {"timeout_steps": a.timeout, "low_water": a.low_water,
                                  **dly.as_dict()}}))


if __name__ == "__main__":
    main()
