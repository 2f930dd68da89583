"""The prefill work list of a plan (host logic, CPU only).

Runtime design §4: the prefill kernel visits only the KV a head can see.  A
plan's prefill items say which KV tiles each CTA visits; these tests read them
back through ``segpaged_plan_prefill_items`` and compare them with the KV
tiles that hold at least one key some row of the item can see, taken from the
oracle's visible sets (``oracle.stored_mask`` over the item's rows).  The
visited set must equal it exactly: no tile a row can see is missed and no
tile that no row can see is visited.  The dense-plus-mask variant must visit
every causal tile instead.  Every (q-head, query row) must belong to exactly
one item.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W


@pytest.fixture(scope="module", autouse=True)
def _lib():
    S.load()


def edge(dtype="bf16", page=64, d=128):
    lens = (1, 2, 63, 129, 200, 300)
    pol = []
    for _ in lens:
        pol += [("global", 0, 0), ("local", 4, 1), ("local", 0, 7), ("local", 70, 3), ("local", 3, 1000),
                ("local", 4, 130)]
    return W.custom("edge", 31, len(lens), 12, 6, d, dtype, page, lens, pol, chunk=140).prefill_problem()


def page_positions(segments, page_size):
    """[first, end) key positions of each page of a head, in page-list order (two int arrays)."""
    out = {}
    for abs_start, length, first, n_pages in segments:
        for i in range(n_pages):
            lo = abs_start + i * page_size
            out[first + i] = (lo, min(abs_start + length, lo + page_size))
    lo = np.array([out[i][0] for i in range(len(out))], np.int64)
    hi = np.array([out[i][1] for i in range(len(out))], np.int64)
    return lo, hi


def inspect(prob, flags=0):
    wl = prob.wl
    p = S.make_problem(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.page_size, wl.dtype,
                       prob.ctx_lens, prob.q_starts, wl.policy, flags=flags)
    plan = S.segpaged_plan_create(p)
    try:
        items = S.segpaged_plan_prefill_items(plan)
        segs = {(b, kv): S.segpaged_plan_head_segments(plan, b, kv)
                for b in range(wl.batch) for kv in range(wl.num_kv_heads)}
        z = S.segpaged_plan_sizes(plan)
    finally:
        S.segpaged_plan_destroy(plan)
    return items, segs, z


CASES = [
    ("tiny-f32", lambda: W.tiny().prefill_problem()),
    ("mistral", lambda: W.mistral().prefill_problem()),
    ("llama", lambda: W.llama().prefill_problem()),  # sequence 0 checked (each sequence has the same shape)
    ("edge-bf16", lambda: edge()),
    ("edge-f32-p16", lambda: edge("f32", 16, 64)),
    ("edge-f32-p64", lambda: edge("f32", 64, 128)),
]


@pytest.mark.parametrize("dense_masked", [False, True])
@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_prefill_items_visit_exactly_the_visible_kv_tiles(name, mk, dense_masked):
    prob = mk()
    wl = prob.wl
    items, segs, z = inspect(prob, S.SP_FLAG_DENSE_MASKED if dense_masked else 0)
    assert len(items) == z.num_prefill_items > 0
    tile = items[0]["tile"]
    assert tile == (128 if wl.dtype == "bf16" else 64)
    ppt = tile // wl.page_size
    covered = {(b, qh): np.zeros(prob.ctx_lens[b], np.int32)
               for b in range(wl.batch) for qh in range(wl.num_q_heads)}
    pages = {h: page_positions(sg, wl.page_size) for h, sg in segs.items()}
    only_b0 = name == "llama"  # the oracle's union of visible sets costs ~7 ms per 128-row tile at 32K
    masks = {}  # the tiles of a GQA group share their rows: one oracle call per (b, kv, rows)
    for it in items:
        b, kv = it["b"], it["kv"]
        if only_b0 and b:
            continue
        L, q0 = prob.ctx_lens[b], prob.q_starts[b]
        kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
        lo, hi = pages[(b, kv)]
        rows = [(it["qh0"], it["q_row0"], it["n_rows0"], it["p0_0"])]
        if it["qh1"] >= 0:
            rows.append((it["qh1"], it["q_row1"], it["n_rows1"], it["p0_1"]))
        p_last = max(r[3] + r[2] - 1 for r in rows)
        see = np.zeros(p_last + 1, bool)
        for qh, q_row, n, p0 in rows:
            assert qh // wl.group == kv and n >= 1
            assert q_row == prob.q_offsets[b] + (p0 - q0) and q0 <= p0 and p0 + n <= L
            covered[(b, qh)][p0:p0 + n] += 1
            # keys the rows p0 .. p0 + n - 1 can see (dense + mask: every causal key)
            if dense_masked:
                see[:p0 + n] = True
            else:
                key = (b, kv, p0, n)
                if key not in masks:
                    masks[key] = oracle.stored_mask(kind, s, w, p0 + n, p0)
                see[:p0 + n] |= masks[key]
        cs = np.concatenate([[0], np.cumsum(see)])
        hits = cs[np.minimum(hi, p_last + 1)] - cs[np.minimum(lo, p_last + 1)] > 0
        needed = set((np.nonzero(hits)[0] // ppt).tolist())
        visited = set(range(it["t0"], it["t1"])) | set(range(it["t2"], it["t3"]))
        assert it["work"] == len(visited) == (it["t1"] - it["t0"]) + (it["t3"] - it["t2"])
        assert visited == needed, (b, kv, rows, sorted(visited ^ needed))
    # every (q-head, query row) once
    for (b, qh), c in covered.items():
        if only_b0 and b:
            continue
        q0 = prob.q_starts[b]
        assert not c[:q0].any() and (c[q0:] == 1).all(), (b, qh)


def test_local_heads_visit_the_sink_and_their_own_window_only():
    """On the 32K layer a LOCAL head stores the sink and the chunk's window run
    (8192 + 4095 positions); each query tile visits the sink tile and the part
    of that run its own rows see, skipping the tiles in between."""
    prob = W.llama().prefill_problem()
    items, segs, _ = inspect(prob)
    wl = prob.wl
    kind = lambda it: wl.policy[it["b"] * wl.num_kv_heads + it["kv"]][0]  # noqa: E731
    local = [it for it in items if kind(it) == "local"]
    glob = [it for it in items if kind(it) == "global"]
    assert local and glob
    head_tiles = -(-sum(sg[3] for sg in segs[(local[0]["b"], local[0]["kv"])]) // 2)
    assert head_tiles >= 96
    # the window run of an item's rows spans 8192 + 127 positions: at most 66 tiles, plus the sink tile
    assert max(it["work"] for it in local) <= 1 + -(-(8192 + 127) // 128) + 1
    assert sum(it["t2"] > it["t1"] for it in local) > len(local) // 2  # a gap after the sink tile
    # a GLOBAL head's last query tile sees the whole causal context: 32768 / 128 tiles
    assert max(it["work"] for it in glob) == 32768 // 128
