"""The oracle's view of a problem's retrieval heads (kept blocks from the same importance inputs)."""
from __future__ import annotations

import oracle


def oracle_head(prob, b: int, kv: int, masses=None):
    """(kind, sink, window, extra) of (b, kv) for the oracle: extra = dict(sel=..., block=...) for a
    retrieval head (its kept blocks chosen by the oracle from the problem's block masses), else {}."""
    wl = prob.wl
    pol = wl.policy[b * wl.num_kv_heads + kv]
    kind, s, w = pol[0], pol[1], pol[2]
    if kind != "retrieval":
        return kind, s, w, {}
    L = prob.ctx_lens[b]
    if w < 0:  # adaptive window, resolved as the planner does
        w = max(1, L // -w)
    masses = masses if masses is not None else prob.block_masses()
    sel = oracle.retrieval_select(L, wl.page_size, s, pol[3], masses[b * wl.num_kv_heads + kv])
    return kind, s, w, dict(sel=sel, block=wl.page_size)
