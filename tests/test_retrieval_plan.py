"""Plans with RETRIEVAL heads (host logic, CPU only).

A retrieval head keeps its sink, its window and the blocks chosen by top-p
importance ("RedKnot head classification", four-kind table, retrieval row:
the whole context as candidates, only the top-p important tokens kept).  The
planner makes its own choice from the same importance inputs as the oracle;
these tests check that the positions a plan stores, its visible-pair ledger
and its prefill work list agree with the oracle's kept blocks and visible sets.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from _retrieval import oracle_head


@pytest.fixture(scope="module", autouse=True)
def _lib():
    S.load()


def _plan(prob, flags=0, masses=None, policy=None):
    wl = prob.wl
    p = S.make_problem(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.page_size, wl.dtype,
                       prob.ctx_lens, prob.q_starts, policy or wl.policy, flags=flags,
                       block_mass=masses if masses is not None else prob.block_masses())
    return S.segpaged_plan_create(p)


def _held(plan, b, kv, L):
    held = np.zeros(L, bool)
    for start, length, _, _ in S.segpaged_plan_head_segments(plan, b, kv):
        assert not held[start:start + length].any()
        held[start:start + length] = True
    return held


def check_plan(prob, flags=0):
    wl = prob.wl
    dense_masked = bool(flags & S.SP_FLAG_DENSE_MASKED)
    plan = _plan(prob, flags)
    try:
        z = S.segpaged_plan_sizes(plan)
        stored = pairs = 0
        for b in range(wl.batch):
            L, q0 = prob.ctx_lens[b], prob.q_starts[b]
            for kv in range(wl.num_kv_heads):
                kind, s, w, extra = oracle_head(prob, b, kv)
                want = oracle.stored_mask("global" if dense_masked else kind, s, w, L, q0, **extra)
                assert np.array_equal(_held(plan, b, kv, L), want), (b, kv)
                stored += int(want.sum())
                pairs += oracle.visible_pairs(kind, s, w, L, q0, **extra)
        assert z.stored_token_heads == stored
        assert z.visible_pairs == pairs * wl.group
    finally:
        S.segpaged_plan_destroy(plan)


def edge_workload(dtype="bf16", page=64, d=128, chunk=140, seed=61):
    lens = (1, 2, 63, 129, 200, 300, 700)
    pol = []
    for _ in lens:
        pol += [("retrieval", 4, 1, 0.5), ("retrieval", 0, 7, 0.9), ("retrieval", 70, 3, 0.3),
                ("retrieval", 3, 1000, 0.7), ("retrieval", 4, 130, 1.0), ("retrieval", 2, 40, 0.0)]
    return W.custom("edge_r", seed, len(lens), 12, 6, d, dtype, page, lens, pol, chunk=chunk)


@pytest.mark.parametrize("name", ["tiny_retrieval", "llama_retrieval"])
@pytest.mark.parametrize("mode", ["decode", "prefill"])
@pytest.mark.parametrize("dense_masked", [False, True])
def test_retrieval_plans_store_the_oracle_sets(name, mode, dense_masked):
    wl = W.ALL[name]()
    if name == "llama_retrieval":
        wl = W.llama_retrieval(batch=2)
    prob = wl.decode_problem() if mode == "decode" else wl.prefill_problem()
    check_plan(prob, S.SP_FLAG_DENSE_MASKED if dense_masked else 0)


@pytest.mark.parametrize("dtype,page,d", [("bf16", 64, 128), ("f32", 16, 64), ("f32", 64, 64)])
@pytest.mark.parametrize("mode", ["decode", "prefill"])
def test_retrieval_edge_policies(dtype, page, d, mode):
    wl = edge_workload(dtype, page, d)
    check_plan(wl.decode_problem() if mode == "decode" else wl.prefill_problem())


def test_retrieval_top_p_one_stores_like_global_and_zero_like_local():
    wl = W.custom("tp", 62, 1, 2, 2, 64, "bf16", 64, (1000,), [("retrieval", 4, 100, 1.0), ("local", 4, 100)],
                  chunk=50)
    for prob in (wl.decode_problem(), wl.prefill_problem()):
        plan = _plan(prob)
        held = _held(plan, 0, 0, 1000)
        S.segpaged_plan_destroy(plan)
        assert held.all()
        pol0 = [("retrieval", 4, 100, 0.0), ("local", 4, 100)]
        plan = _plan(prob, policy=pol0)
        a, b = _held(plan, 0, 0, 1000), _held(plan, 0, 1, 1000)
        S.segpaged_plan_destroy(plan)
        assert np.array_equal(a, b)


def test_retrieval_prefill_items_visit_every_visible_tile():
    """Every KV tile holding a key some row of an item sees is visited; visited tiles lie between the
    first and the last such tile; every (q-head, row) belongs to exactly one item."""
    for wl in (edge_workload(), edge_workload("f32", 16, 64), W.llama_retrieval(batch=1)):
        prob = wl.prefill_problem()
        plan = _plan(prob)
        try:
            items = S.segpaged_plan_prefill_items(plan)
            cover = {}
            for it in items:
                b, kv, T = it["b"], it["kv"], it["tile"]
                L, q0 = prob.ctx_lens[b], prob.q_starts[b]
                kind, s, w, extra = oracle_head(prob, b, kv)
                ppt = T // wl.page_size
                segs = S.segpaged_plan_head_segments(plan, b, kv)
                page_of = {}
                for start, length, first, npages in segs:
                    for j in range(length):
                        page_of[start + j] = first + j // wl.page_size
                seen = set()
                for x in (0, 1):
                    if x == 1 and it["qh1"] < 0:
                        continue
                    p0, n = it["p0_%d" % x], it["n_rows%d" % x]
                    for r in range(n):
                        key = (b, it["qh%d" % x], p0 - q0 + r)
                        cover[key] = cover.get(key, 0) + 1
                    if kind != "retrieval":
                        continue
                    # keys some row p0 .. p0 + n - 1 sees: the stored set of a call with exactly those queries
                    for j in np.flatnonzero(oracle.stored_mask(kind, s, w, p0 + n, p0, **extra)):
                        seen.add(page_of[int(j)] // ppt)
                visited = set(range(it["t0"], it["t1"])) | set(range(it["t2"], it["t3"]))
                assert seen <= visited, (b, kv, sorted(seen - visited))
                if seen:
                    assert min(visited) >= min(seen) and max(visited) <= max(seen)
            assert all(c == 1 for c in cover.values())
            assert len(cover) == prob.total_queries * wl.num_q_heads
        finally:
            S.segpaged_plan_destroy(plan)


def test_retrieval_argument_checks():
    wl = W.tiny_retrieval()
    prob = wl.decode_problem()
    lib = S.load()

    def status(policy=None, masses="default", flags=0):
        m = prob.block_masses() if masses == "default" else masses
        p = S.make_problem(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.page_size, wl.dtype,
                           prob.ctx_lens, prob.q_starts, policy or wl.policy, flags=flags, block_mass=m)
        st, plan = S.segpaged_plan_create_status(p)
        if plan:
            S.segpaged_plan_destroy(plan)
        return st

    assert status() == S.SP_OK
    assert status(masses=None) == S.SP_ERR_INVALID_ARG
    assert status(masses=[None, None]) == S.SP_ERR_INVALID_ARG
    bad = prob.block_masses()
    bad[1] = list(bad[1])
    bad[1][3] = -1.0
    assert status(masses=bad) == S.SP_ERR_INVALID_ARG and "block_mass" in S.last_error()
    bad[1][3] = float("nan")
    assert status(masses=bad) == S.SP_ERR_INVALID_ARG
    assert status(policy=[("global", 0, 0), ("retrieval", 4, 32, float("nan"))]) == S.SP_ERR_INVALID_ARG
    assert status(policy=[("global", 0, 0), ("retrieval", -1, 32, 0.5)]) == S.SP_ERR_INVALID_ARG
    assert status(policy=[("global", 0, 0), ("retrieval", 4, 0, 0.5)]) == S.SP_ERR_INVALID_ARG
    assert status(flags=S.SP_FLAG_RING) == S.SP_ERR_UNSUPPORTED
    assert lib is not None
