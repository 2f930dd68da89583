"""Brute-force checker for the oracle on tiny inputs (test infrastructure only).

It enumerates each query's visible set as a Python set built from the words
of the head-kind definitions, not from the oracle's predicate:

* a global (or dense) head sees every position up to and including the query
  ("SegPagedAttention runtime design", §1; "RedKnot head classification",
  four-kind table);
* a local head sees the sequence's first ``sink`` tokens and its ``window``
  most recent tokens, the query's own token being the most recent one
  ("SegPagedAttention runtime design", §1 and §3).

Softmax sums use ``math.fsum`` (exactly rounded) and ``math.exp``.
"""
from __future__ import annotations

import math


def visible_positions(kind: str, sink: int, window: int, p: int) -> list[int]:
    if kind in ("global", "dense"):
        return list(range(p + 1))
    first_tokens = {j for j in range(sink) if j <= p}
    most_recent = {p - back for back in range(window) if p - back >= 0}
    return sorted(first_tokens | most_recent)


def attention_row(q, k, v, kind: str, sink: int, window: int, p: int, scale: float):
    """One row: lists of floats in, (out list, lse) out."""
    vis = visible_positions(kind, sink, window, p)
    scores = [scale * math.fsum(a * b for a, b in zip(q, k[j])) for j in vis]
    m = max(scores)
    w = [math.exp(s - m) for s in scores]
    z = math.fsum(w)
    d = len(q)
    out = [math.fsum(w[i] * v[j][t] for i, j in enumerate(vis)) / z for t in range(d)]
    return out, m + math.log(z)


def stored_positions(kind: str, sink: int, window: int, L: int, q0: int) -> set[int]:
    """Union of the visible sets of queries q0 .. L-1."""
    keep: set[int] = set()
    for p in range(q0, L):
        keep |= set(visible_positions(kind, sink, window, p))
    return keep
