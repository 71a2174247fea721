"""Splitting a batch of requests into two micro-batches.

Two-micro-batch overlap runs ub0's communication while ub1 computes and the
reverse, so the two halves should carry the same number of tokens.  Splitting
at request boundaries leaves them uneven (three requests of 7003, 6928 and 2453
tokens give 7003 / 9381, 1.34x); splitting at the token midpoint cuts one
request in two and gives 8192 / 8192 (DP Attention and TBO for DeepSeek-V4 on
MI355X, §TBOのマイクロバッチ分割改善).  The second piece of a cut request then
treats the first piece's tokens as its prefix.

A micro-batch is a list of (request index, first token, token count) pieces.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

Piece = Tuple[int, int, int]


def split_at_request_boundary(lengths: Sequence[int]) -> Tuple[List[Piece], List[Piece]]:
    """Whole requests only: the first micro-batch takes requests while it stays at
    or below half of the tokens, and always at least one request."""
    total = sum(lengths)
    ub0: List[Piece] = []
    used = 0
    for i, n in enumerate(lengths):
        if ub0 and used + n > total / 2:
            break
        ub0.append((i, 0, n))
        used += n
    ub1 = [(i, 0, n) for i, n in enumerate(lengths)][len(ub0):]
    return ub0, ub1


def split_even(lengths: Sequence[int]) -> Tuple[List[Piece], List[Piece]]:
    """Token-midpoint split: ub0 gets the first floor(total/2) tokens, ub1 the
    rest; the request that straddles the midpoint is cut in two."""
    total = sum(lengths)
    half = total // 2
    ub0: List[Piece] = []
    ub1: List[Piece] = []
    pos = 0
    for i, n in enumerate(lengths):
        if pos + n <= half:
            ub0.append((i, 0, n))
        elif pos >= half:
            ub1.append((i, 0, n))
        else:
            cut = half - pos
            ub0.append((i, 0, cut))
            ub1.append((i, cut, n - cut))
        pos += n
    return ub0, ub1


def tokens(ub: Sequence[Piece]) -> int:
    return sum(p[2] for p in ub)


def token_ranges(lengths: Sequence[int], ub: Sequence[Piece]) -> List[Tuple[int, int]]:
    """Row ranges [start, end) of a micro-batch's pieces in the concatenated batch."""
    starts = [0]
    for n in lengths:
        starts.append(starts[-1] + n)
    return [(starts[i] + first, starts[i] + first + count) for i, first, count in ub]
