"""The decode work split of a plan (host logic, CPU only).

A decode plan cuts the concatenated page lists of all (sequence, kv-head)
pairs into balanced CTA ranges, at head boundaries; a head cut into several
items gets one partial slot per item and an arrival counter, and on bf16
pages a head cut into more than 16 items also gets merge groups of
ceil(sqrt(n)) slots, each with a group slot and a counter.  These tests read
the split back through ``segpaged_plan_decode_items`` and check it against
those rules and against the plan's workspace size.
"""
from __future__ import annotations

import math
from collections import defaultdict

import pytest

from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W

DEFAULT_CTAS = 2 * 148
ONE_LEVEL_MAX = 16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    S.load()


def make_plan(prob, **kw):
    wl = prob.wl
    p = S.make_problem(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.page_size, wl.dtype,
                       prob.ctx_lens, prob.q_starts, wl.policy, **kw)
    return S.segpaged_plan_create(p)


def edge(g=16, d=128):
    lens = (1, 2, 63, 64, 65, 129, 300)
    pol = []
    for _ in lens:
        pol += [("global", 0, 0), ("local", 4, 1), ("local", 0, 7), ("local", 70, 3), ("dense", 0, 0)]
    return W.custom("edge", 21, len(lens), 5 * g, 5, d, "bf16", 64, lens, pol).decode_problem()


CASES = [
    ("mistral", lambda: W.mistral().decode_problem(), {}),
    ("mistral-1cta", lambda: W.mistral().decode_problem(), {"target_ctas": 1}),
    ("mistral-7", lambda: W.mistral().decode_problem(), {"target_ctas": 7}),
    ("mistral-150", lambda: W.mistral().decode_problem(), {"target_ctas": 150}),
    ("mistral-1000", lambda: W.mistral().decode_problem(), {"target_ctas": 1000}),
    ("mistral-e4m3", lambda: W.mistral().decode_problem(), {"kv_dtype": "e4m3", "k_scale": 0.02, "v_scale": 0.02}),
    ("llama", lambda: W.llama().decode_problem(), {}),
    ("ragged", lambda: W.ragged().decode_problem(), {}),
    ("mha", lambda: W.mha().decode_problem(), {}),
    ("tiny-f32", lambda: W.tiny().decode_problem(), {}),
    ("edge-g16", lambda: edge(16, 128), {}),
    ("edge-g1-d64", lambda: edge(1, 64), {}),
    ("ring", lambda: W.mistral().decode_problem(), {"flags": S.SP_FLAG_RING, "append_capacity": 64}),
]


@pytest.mark.parametrize("name,mk,kw", CASES, ids=[c[0] for c in CASES])
def test_decode_split_follows_its_rules(name, mk, kw):
    prob = mk()
    wl = prob.wl
    plan = make_plan(prob, **kw)
    try:
        z = S.segpaged_plan_sizes(plan)
        items = S.segpaged_plan_decode_items(plan)
        n_ctas = z.num_decode_ctas
        pages = {(b, kv): len(S.segpaged_plan_head_pages(plan, b, kv))
                 for b in range(wl.batch) for kv in range(wl.num_kv_heads)}
    finally:
        S.segpaged_plan_destroy(plan)
    total_pages = sum(pages.values())
    assert n_ctas == min(kw.get("target_ctas") or DEFAULT_CTAS, total_pages)

    # CTAs in launch order.  A head's first page costs 4.5 pages (the page and
    # the head start), so when a CTA's share is below that a cut can fall
    # inside it and leave a CTA empty (the kernels return at once from such a
    # CTA).
    ctas = [it["cta"] for it in items]
    assert ctas == sorted(ctas) and set(ctas) <= set(range(n_ctas))

    # every head's pages are covered once, in order, by consecutive items
    by_head = defaultdict(list)
    order = []
    for i, it in enumerate(items):
        h = (it["b"], it["kv"])
        if not order or order[-1] != h:
            assert h not in by_head, f"items of {h} are not consecutive"
            order.append(h)
        by_head[h].append(it)
    assert set(by_head) == set(pages)
    for h, its in by_head.items():
        assert its[0]["page_begin"] == 0 and its[-1]["page_end"] == pages[h]
        for a, c in zip(its, its[1:]):
            assert a["page_end"] == c["page_begin"]
        assert all(it["page_end"] > it["page_begin"] for it in its)

    # balance, in hundredths of a page as the planner costs them: 100 per page
    # and 350 more for the page that starts a head.  Each CTA's range ends at
    # the first page whose running cost reaches its equal share, so it exceeds
    # that share by less than its last page's cost: at most 450.
    cost = defaultdict(int)
    for it in items:
        cost[it["cta"]] += 100 * (it["page_end"] - it["page_begin"]) + (350 if it["page_begin"] == 0 else 0)
    total_cost = sum(cost.values())
    assert total_cost == 100 * total_pages + 350 * len(pages)
    assert max(cost.values()) <= -(-total_cost // n_ctas) + 450

    # slots, counters and merge groups
    two_level_pages = wl.dtype == "bf16" and kw.get("kv_dtype") in (None, "bf16")
    item_slots, group_slots, counters = [], [], []
    for h, its in by_head.items():
        n = len(its)
        if n == 1:
            it = its[0]
            assert (it["slot"], it["counter"], it["group_size"], it["group_counter"]) == (-1, -1, 0, -1)
            continue
        slot0 = its[0]["slot0"]
        assert [it["slot"] for it in its] == list(range(slot0, slot0 + n))
        assert all(it["n_slots"] == n and it["slot0"] == slot0 for it in its)
        assert len({it["counter"] for it in its}) == 1
        item_slots += [it["slot"] for it in its]
        counters.append(its[0]["counter"])
        gsz = its[0]["group_size"]
        if two_level_pages and n > ONE_LEVEL_MAX:
            assert gsz == math.isqrt(n - 1) + 1  # ceil(sqrt(n))
            ng = -(-n // gsz)
            g0 = its[0]["group_slot0"]
            group_slots += list(range(g0, g0 + ng))
            gcs = [it["group_counter"] for it in its]
            # items of group j share its counter; groups have distinct counters
            for j in range(ng):
                assert len(set(gcs[j * gsz:(j + 1) * gsz])) == 1
            assert len(set(gcs)) == ng
            counters += sorted(set(gcs))
        else:
            assert gsz == 0 and all(it["group_counter"] == -1 for it in its)
    all_slots = item_slots + group_slots
    assert sorted(all_slots) == list(range(len(all_slots)))  # no gap, no overlap
    assert sorted(counters) == list(range(len(counters)))
    if not two_level_pages:
        assert not group_slots

    # the workspace holds the status block, the counters and every slot
    r256 = lambda x: -(-x // 256) * 256  # noqa: E731
    slot_bytes = wl.group * (wl.head_dim + 4) * 4
    assert z.workspace_bytes == 256 + r256(4 * len(counters)) + r256(slot_bytes * len(all_slots))


def test_heads_split_into_many_items_merge_in_two_levels():
    """The 8K layer at 1000 CTAs cuts its GLOBAL heads into about a hundred items."""
    plan = make_plan(W.mistral().decode_problem(), target_ctas=1000)
    try:
        items = S.segpaged_plan_decode_items(plan)
    finally:
        S.segpaged_plan_destroy(plan)
    sizes = {it["n_slots"]: it["group_size"] for it in items if it["slot"] >= 0}
    assert max(sizes) > 64
    assert all(g == (math.isqrt(n - 1) + 1 if n > ONE_LEVEL_MAX else 0) for n, g in sizes.items())


def test_prefill_plans_have_no_decode_items():
    plan = make_plan(W.tiny().prefill_problem())
    try:
        assert S.segpaged_plan_decode_items(plan) == []
    finally:
        S.segpaged_plan_destroy(plan)
