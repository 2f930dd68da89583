"""Brute-force checker for the oracle on tiny inputs (test infrastructure only).

It enumerates each query's visible set as a Python set built from the words
of the head-kind definitions, not from the oracle's predicate:

* a global (or dense) head sees every position up to and including the query
  ("SegPagedAttention runtime design", §1; "RedKnot head classification",
  four-kind table);
* a local head sees the sequence's first ``sink`` tokens and its ``window``
  most recent tokens, the query's own token being the most recent one
  ("SegPagedAttention runtime design", §1 and §3);
* a retrieval head sees what a local head sees plus every earlier position
  of the blocks it keeps; it keeps the fewest blocks whose importance
  reaches the fraction ``top_p`` of the total ("RedKnot head classification",
  four-kind table: full KV, only the top-p important tokens kept), found
  here by trying every set of blocks, smallest sets first.

Softmax sums use ``math.fsum`` (exactly rounded) and ``math.exp``.
"""
from __future__ import annotations

import itertools
import math


def visible_positions(kind: str, sink: int, window: int, p: int, kept_blocks=(), block: int = 1) -> list[int]:
    if kind in ("global", "dense"):
        return list(range(p + 1))
    first_tokens = {j for j in range(sink) if j <= p}
    most_recent = {p - back for back in range(window) if p - back >= 0}
    kept = set()
    if kind == "retrieval":
        kept = {j for i in kept_blocks for j in range(i * block, (i + 1) * block) if j <= p}
    return sorted(first_tokens | most_recent | kept)


def kept_blocks(L: int, block: int, sink: int, top_p: float, mass) -> set[int]:
    """Blocks a retrieval head keeps, by exhaustive search (tiny inputs only).

    Candidates are the blocks holding some position >= sink.  Among all sets of candidates,
    take the smallest size k for which some set's importance reaches top_p of the total
    (every candidate when top_p >= 1, none when top_p <= 0); of the sets of that size take
    the one with the largest importance, and among equals the one whose blocks, listed in
    decreasing importance (lower block first on ties), come earliest.
    """
    n = -(-L // block)
    cand = [i for i in range(n) if (i + 1) * block > sink]
    if top_p >= 1:
        return set(cand)
    if top_p <= 0:
        return set()
    total = math.fsum(mass[i] for i in cand)
    target = top_p * total
    for k in range(len(cand) + 1):
        best = None
        for sub in itertools.combinations(cand, k):
            m = math.fsum(mass[i] for i in sub)
            if m < target:
                continue
            key = (-m, sorted(sub, key=lambda i: (-mass[i], i)))
            if best is None or key < best[0]:
                best = (key, set(sub))
        if best is not None:
            return best[1]
    return set(cand)


def attention_row(q, k, v, kind: str, sink: int, window: int, p: int, scale: float, kept=(), block: int = 1):
    """One row: lists of floats in, (out list, lse) out."""
    vis = visible_positions(kind, sink, window, p, kept, block)
    scores = [scale * math.fsum(a * b for a, b in zip(q, k[j])) for j in vis]
    m = max(scores)
    w = [math.exp(s - m) for s in scores]
    z = math.fsum(w)
    d = len(q)
    out = [math.fsum(w[i] * v[j][t] for i, j in enumerate(vis)) / z for t in range(d)]
    return out, m + math.log(z)


def stored_positions(kind: str, sink: int, window: int, L: int, q0: int, kept=(), block: int = 1) -> set[int]:
    """Union of the visible sets of queries q0 .. L-1."""
    keep: set[int] = set()
    for p in range(q0, L):
        keep |= set(visible_positions(kind, sink, window, p, kept, block))
    return keep
