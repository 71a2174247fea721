"""The micro-batch planner against the split the pages print (three requests of
7003, 6928 and 2453 tokens: 7003 / 9381 at request boundaries, 8192 / 8192 at the
token midpoint) and against invariants on random request mixes."""
import json
import os

import numpy as np

from mixture_experts_fp32_b200 import microbatch as mb

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def test_page_example():
    f = json.load(open(GOLDEN))["microbatch_split"]
    ub0, ub1 = mb.split_at_request_boundary(f["requests"])
    assert [mb.tokens(ub0), mb.tokens(ub1)] == f["boundary_split"]
    assert round(mb.tokens(ub1) / mb.tokens(ub0), 2) == f["boundary_ratio"]
    ub0, ub1 = mb.split_even(f["requests"])
    assert [mb.tokens(ub0), mb.tokens(ub1)] == f["even_split"]
    # the second request is cut: its tail starts ub1 where its head ended ub0
    assert ub0[-1][0] == ub1[0][0] == 1
    assert ub0[-1][1] + ub0[-1][2] == ub1[0][1]


def test_even_split_invariants():
    rng = np.random.default_rng(0)
    for _ in range(200):
        lengths = list(rng.integers(1, 5000, size=rng.integers(1, 9)))
        ub0, ub1 = mb.split_even(lengths)
        total = sum(lengths)
        assert mb.tokens(ub0) == total // 2 and mb.tokens(ub1) == total - total // 2
        ranges = mb.token_ranges(lengths, ub0) + mb.token_ranges(lengths, ub1)
        covered = np.zeros(total, dtype=int)
        for a, b in ranges:
            covered[a:b] += 1
        assert (covered == 1).all()              # every token exactly once, in order
        assert all(r[0] < r[1] for r in ranges)
        b0, b1 = mb.split_at_request_boundary(lengths)
        assert mb.tokens(b0) + mb.tokens(b1) == total
        assert abs(mb.tokens(ub0) - mb.tokens(ub1)) <= abs(mb.tokens(b0) - mb.tokens(b1))
