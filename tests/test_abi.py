"""C-ABI library and host planner tests (no GPU: only host-side entry points run)."""
from __future__ import annotations

import ctypes
import re
from pathlib import Path

import numpy as np
import pytest

import oracle
from head_aware_paged_build_b200 import build_ext
from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W

ROOT = Path(__file__).resolve().parent.parent


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_ext.build()
    return S.load()


def header_symbols():
    text = (ROOT / "include" / "segpaged.h").read_text()
    return re.findall(r"SP_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_library_exports_every_header_symbol():
    names = header_symbols()
    assert len(names) == len(S.EXPORTED) and set(names) == set(S.EXPORTED)
    lib = S.load()
    for n in names:
        assert getattr(lib, n) is not None
    assert S.segpaged_abi_version() == 2
    assert S.status_name(S.SP_ERR_WORKSPACE) == "SP_ERR_WORKSPACE"


def plan_for(prob, **kw):
    wl = prob.wl
    p = S.make_problem(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.page_size, wl.dtype,
                       prob.ctx_lens, prob.q_starts, wl.policy, **kw)
    return S.segpaged_plan_create(p), p


def oracle_stored(prob, dense_masked=False):
    wl = prob.wl
    n = 0
    for b in range(wl.batch):
        for kv in range(wl.num_kv_heads):
            kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
            if dense_masked:
                kind = "global"
            n += int(oracle.stored_mask(kind, s, w, prob.ctx_lens[b], prob.q_starts[b]).sum())
    return n


@pytest.mark.parametrize("name", ["tiny", "mistral"])
@pytest.mark.parametrize("mode", ["decode", "prefill"])
def test_plan_sizes_match_oracle(name, mode):
    wl = W.ALL[name]()
    prob = wl.decode_problem() if mode == "decode" else wl.prefill_problem()
    plan, _ = plan_for(prob)
    try:
        z = S.segpaged_plan_sizes(plan)
        assert z.stored_token_heads == oracle_stored(prob)
        assert z.dense_token_heads == sum(prob.ctx_lens) * wl.num_kv_heads
        pairs = 0
        for b in range(wl.batch):
            for kv in range(wl.num_kv_heads):
                kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
                pairs += oracle.visible_pairs(kind, s, w, prob.ctx_lens[b], prob.q_starts[b])
        assert z.visible_pairs == pairs * wl.group
        assert z.is_decode == (mode == "decode")
        assert z.num_queries == prob.total_queries
        elem = 2 if wl.dtype == "bf16" else 4
        assert z.page_bytes == wl.page_size * wl.head_dim * elem
        assert z.workspace_bytes >= 256 and z.workspace_bytes % 256 == 0
    finally:
        S.segpaged_plan_destroy(plan)


def test_plan_sizes_of_large_layers_closed_form():
    """Llama-70B-shaped: 721,120 stored token-heads at decode, 950,440 for the 4096-query chunk."""
    for prob, want in ((W.llama().decode_problem(), 721_120), (W.llama().prefill_problem(), 950_440),
                       (W.mha().decode_problem(), 4 * (8 * 131072 + 56 * 132))):
        plan, _ = plan_for(prob)
        z = S.segpaged_plan_sizes(plan)
        assert z.stored_token_heads == want
        S.segpaged_plan_destroy(plan)
    wl = W.llama()
    plan, _ = plan_for(wl.prefill_problem())
    z = S.segpaged_plan_sizes(plan)
    # visible FLOPs of the 4096-query chunk: 4 d sum |V(p)| = 1.1824e13
    assert 4 * 128 * z.visible_pairs == pytest.approx(1.1824e13, rel=1e-4)
    S.segpaged_plan_destroy(plan)


def _random_policy_cases(n=60, seed=0):
    rng = np.random.default_rng(seed)
    for _ in range(n):
        L = int(rng.integers(1, 300))
        q0 = int(rng.integers(0, L))
        kind = ["global", "local", "dense"][int(rng.integers(0, 3))]
        s = int(rng.integers(0, 40))
        w = int(rng.integers(1, 120))
        yield L, q0, kind, s, w


@pytest.mark.parametrize("page", [16, 64])
@pytest.mark.parametrize("dense_masked", [False, True])
def test_segments_hold_exactly_the_oracle_stored_set(page, dense_masked):
    for L, q0, kind, s, w in _random_policy_cases(seed=page + dense_masked):
        p = S.make_problem(1, 1, 1, 64, page, "f32", [L], [q0], [(kind, s, w)],
                           flags=S.SP_FLAG_DENSE_MASKED if dense_masked else 0)
        plan = S.segpaged_plan_create(p)
        segs = S.segpaged_plan_head_segments(plan, 0, 0)
        pages = S.segpaged_plan_head_pages(plan, 0, 0)
        S.segpaged_plan_destroy(plan)
        held = np.zeros(L, bool)
        next_page = 0
        for start, length, first_page, npages in segs:
            assert length >= 1 and not held[start:start + length].any()
            held[start:start + length] = True
            assert first_page == next_page and npages == -(-length // page)
            next_page += npages
        assert len(pages) == next_page
        want = oracle.stored_mask("global" if dense_masked else kind, s, w, L, q0)
        assert np.array_equal(held, want), (L, q0, kind, s, w, segs)


def test_page_ids_first_page_and_permutation():
    wl = W.tiny()
    prob = wl.decode_problem()
    plan, _ = plan_for(prob)
    n = S.segpaged_plan_sizes(plan).num_pages
    S.segpaged_plan_destroy(plan)
    perm = list(np.random.default_rng(3).permutation(n))
    plan, _ = plan_for(prob, first_page=7, page_ids=perm)
    z = S.segpaged_plan_sizes(plan)
    assert z.pool_pages == 7 + n and z.num_pages == n
    got = S.segpaged_plan_head_pages(plan, 0, 0) + S.segpaged_plan_head_pages(plan, 0, 1)
    assert got == [7 + int(x) for x in perm]
    S.segpaged_plan_destroy(plan)
    bad = S.make_problem(1, 4, 2, 64, 16, "f32", prob.ctx_lens, prob.q_starts, wl.policy,
                         page_ids=[0] * n)
    st, _ = S.segpaged_plan_create_status(bad)
    assert st == S.SP_ERR_INVALID_ARG and "distinct" in S.last_error()


BASE = dict(batch=1, num_q_heads=4, num_kv_heads=2, head_dim=64, page_size=16, dtype="f32", ctx_len=[100],
            q_start=[99], policy=[("global", 0, 0), ("local", 4, 8)])


@pytest.mark.parametrize("change,code", [
    (dict(batch=0, ctx_len=[], q_start=[], policy=[]), S.SP_ERR_INVALID_ARG),
    (dict(ctx_len=[0], q_start=[0]), S.SP_ERR_INVALID_ARG),
    (dict(q_start=[100]), S.SP_ERR_INVALID_ARG),
    (dict(q_start=[-1]), S.SP_ERR_INVALID_ARG),
    (dict(policy=[("global", 0, 0), ("local", 4, 0)]), S.SP_ERR_INVALID_ARG),
    (dict(policy=[("global", 0, 0), ("local", -1, -2)]), S.SP_ERR_INVALID_ARG),
    (dict(policy=[("global", 0, 0), ("local", -1, 8)]), S.SP_ERR_INVALID_ARG),
    (dict(policy=[("global", 0, 0), (7, 0, 8)]), S.SP_ERR_INVALID_ARG),
    (dict(policy=[("global", 0, 0), ("retrieval", 4, 8, 0.5)]), S.SP_ERR_INVALID_ARG),  # no block_mass
    (dict(head_dim=96), S.SP_ERR_UNSUPPORTED),
    (dict(dtype=5), S.SP_ERR_UNSUPPORTED),
    (dict(dtype="bf16"), S.SP_ERR_UNSUPPORTED),  # bf16 needs page 64
    (dict(page_size=32), S.SP_ERR_UNSUPPORTED),
    (dict(num_q_heads=5), S.SP_ERR_UNSUPPORTED),
    (dict(num_q_heads=34, num_kv_heads=2), S.SP_ERR_UNSUPPORTED),
])
def test_plan_validation_errors(change, code):
    args = dict(BASE)
    args.update(change)
    p = S.make_problem(**args)
    st, plan = S.segpaged_plan_create_status(p)
    assert st == code, S.last_error()
    assert not plan
    assert S.last_error()


def test_unknown_flag_and_negative_first_page_rejected():
    for kw in (dict(flags=4), dict(first_page=-1), dict(target_ctas=-2)):
        p = S.make_problem(**BASE, **kw)
        st, _ = S.segpaged_plan_create_status(p)
        assert st == S.SP_ERR_INVALID_ARG


def test_decode_split_uses_target_ctas():
    wl = W.mistral()
    prob = wl.decode_problem()
    for target, want in ((0, 296), (10, 10), (100000, None)):
        plan, _ = plan_for(prob, target_ctas=target)
        z = S.segpaged_plan_sizes(plan)
        assert z.num_decode_ctas == (want if want is not None else z.num_pages)
        S.segpaged_plan_destroy(plan)


def test_device_calls_reject_bad_arguments_before_launch():
    """Host-side checks run before any CUDA call, so they work without a GPU."""
    wl = W.tiny()
    plan, _ = plan_for(wl.decode_problem())
    z = S.segpaged_plan_sizes(plan)
    lib = S.load()
    # NULL table / misaligned pointers / short workspace never reach CUDA
    assert lib.segpaged_attention(plan, None, 16, 16, 16, 16, None, 0.0, 256, z.workspace_bytes, None) \
        == S.SP_ERR_INVALID_ARG
    assert lib.segpaged_attention(plan, 256, 16, 16, 16, 16, None, 0.0, 256, 1, None) == S.SP_ERR_WORKSPACE
    assert lib.segpaged_attention(plan, 256, 16, 16, 17, 16, None, 0.0, 256, z.workspace_bytes, None) \
        == S.SP_ERR_INVALID_ARG
    assert lib.segpaged_attention(plan, 256, 16, 16, 16, 16, None, float("nan"), 256, z.workspace_bytes, None) \
        == S.SP_ERR_INVALID_ARG
    assert lib.build_segpaged_cache(plan, 256, 16, 16, -5, 0, 64, 16, 16, None) == S.SP_ERR_INVALID_ARG
    assert lib.build_segpaged_cache(plan, 256, 16, 16, 0, 0, 3, 16, 16, None) == S.SP_ERR_INVALID_ARG
    assert lib.segpaged_table_write(plan, 256, 8, None) == S.SP_ERR_WORKSPACE
    S.segpaged_plan_destroy(plan)


@pytest.mark.parametrize("div", [1, 2, 3, 7])
def test_adaptive_window_resolves_per_sequence(div):
    """window = -div selects max(1, L // div) per sequence (adaptive window of the head-classification page)."""
    lens = [1, 5, 64, 100, 1000, 4097]
    pol = []
    for _ in lens:
        pol += [("local", 4, -div), ("global", 0, 0)]
    for mode in ("decode", "prefill"):
        q0 = [L - 1 if mode == "decode" else max(0, L - 37) for L in lens]
        p = S.make_problem(len(lens), 2, 2, 64, 16, "f32", lens, q0, pol)
        plan = S.segpaged_plan_create(p)
        for b, L in enumerate(lens):
            segs = S.segpaged_plan_head_segments(plan, b, 0)
            held = np.zeros(L, bool)
            for start, length, _, _ in segs:
                held[start:start + length] = True
            want = oracle.stored_mask("local", 4, max(1, L // div), L, q0[b])
            assert np.array_equal(held, want), (b, L, div)
        S.segpaged_plan_destroy(plan)


@pytest.mark.parametrize("page", [16, 64])
def test_ring_plan_layout(page):
    """Ring plans hold the same stored set; GLOBAL heads reserve pages, LOCAL heads a ring of ceil(w/P)+1 pages."""
    rng = np.random.default_rng(page)
    for _ in range(40):
        L = int(rng.integers(1, 400))
        s = int(rng.integers(0, 70))
        w = int(rng.integers(1, 150))
        cap = int(rng.integers(0, 200))
        p = S.make_problem(1, 2, 2, 64, page, "f32", [L], [L - 1], [("local", s, w), ("global", 0, 0)],
                           flags=S.SP_FLAG_RING, append_capacity=cap)
        plan = S.segpaged_plan_create(p)
        held = np.zeros(L, bool)
        for start, length, _, _ in S.segpaged_plan_head_segments(plan, 0, 0):
            held[start:start + length] = True
        assert np.array_equal(held, oracle.stored_mask("local", s, w, L, L - 1))
        assert len(S.segpaged_plan_head_pages(plan, 0, 0)) == -(-s // page) + (-(-w // page) + 1)
        assert len(S.segpaged_plan_head_pages(plan, 0, 1)) == -(-(L + cap) // page)
        assert S.segpaged_plan_sizes(plan).stored_token_heads == int(held.sum()) + L
        S.segpaged_plan_destroy(plan)


def test_ring_plan_validation():
    base = dict(batch=1, num_q_heads=2, num_kv_heads=2, head_dim=64, page_size=16, dtype="f32", ctx_len=[100],
                policy=[("local", 4, 8), ("global", 0, 0)])
    for kw, code in ((dict(q_start=[90], flags=S.SP_FLAG_RING), S.SP_ERR_UNSUPPORTED),
                     (dict(q_start=[99], flags=S.SP_FLAG_RING | S.SP_FLAG_DENSE_MASKED), S.SP_ERR_UNSUPPORTED),
                     (dict(q_start=[99], append_capacity=5), S.SP_ERR_INVALID_ARG),
                     (dict(q_start=[99], flags=S.SP_FLAG_RING, append_capacity=-1), S.SP_ERR_INVALID_ARG)):
        st, _ = S.segpaged_plan_create_status(S.make_problem(**base, **kw))
        assert st == code, (kw, S.last_error())
    # appends need a ring plan (host-side check, no launch)
    plan = S.segpaged_plan_create(S.make_problem(**base, q_start=[99]))
    assert S.load().segpaged_decode_append(plan, 256, 16, 16, 0, 0, 16, 16, 256, None) == S.SP_ERR_INVALID_ARG
    S.segpaged_plan_destroy(plan)


def test_e4m3_pages_plan_and_validation():
    """E4M3 pages: 1-byte pages for bf16 decode plans; everything else is rejected before any launch."""
    base = dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=64, dtype="bf16",
                ctx_len=[300, 77], q_start=[299, 76], policy=[("global", 0, 0), ("local", 4, 64)] * 2)
    plan = S.segpaged_plan_create(S.make_problem(**base, kv_dtype="e4m3", k_scale=0.5, v_scale=2.0))
    ref = S.segpaged_plan_create(S.make_problem(**base))
    z, zr = S.segpaged_plan_sizes(plan), S.segpaged_plan_sizes(ref)
    assert z.page_bytes == 64 * 128 and zr.page_bytes == 2 * 64 * 128
    assert (z.num_pages, z.stored_token_heads, z.visible_pairs) == (zr.num_pages, zr.stored_token_heads,
                                                                   zr.visible_pairs)
    S.segpaged_plan_destroy(plan)
    S.segpaged_plan_destroy(ref)
    # the problem dtype as kv_dtype is the default layout
    plan = S.segpaged_plan_create(S.make_problem(**base, kv_dtype="bf16"))
    assert S.segpaged_plan_sizes(plan).page_bytes == 2 * 64 * 128
    S.segpaged_plan_destroy(plan)
    prefill = dict(base, q_start=[0, 0])
    for kw, code in ((dict(base, kv_dtype="e4m3", k_scale=0.0), S.SP_ERR_INVALID_ARG),
                     (dict(base, kv_dtype="e4m3", v_scale=-1.0), S.SP_ERR_INVALID_ARG),
                     (dict(base, kv_dtype="e4m3", k_scale=float("inf")), S.SP_ERR_INVALID_ARG),
                     (dict(base, kv_dtype="e4m3", v_scale=float("nan")), S.SP_ERR_INVALID_ARG),
                     (dict(base, kv_dtype=9), S.SP_ERR_UNSUPPORTED),
                     (dict(prefill, kv_dtype="e4m3"), S.SP_ERR_UNSUPPORTED),
                     (dict(BASE, kv_dtype="e4m3"), S.SP_ERR_UNSUPPORTED)):  # fp32 queries
        st, pl = S.segpaged_plan_create_status(S.make_problem(**kw))
        assert st == code and not pl, (kw, S.last_error())


def test_multi_layer_build_checks_before_launch():
    base = dict(batch=1, num_q_heads=4, num_kv_heads=2, head_dim=64, page_size=64, dtype="bf16", ctx_len=[300],
                q_start=[299], policy=[("global", 0, 0), ("local", 4, 64)])
    a = S.segpaged_plan_create(S.make_problem(**base))
    b = S.segpaged_plan_create(S.make_problem(**dict(base, head_dim=128)))
    lib = S.load()
    arr = lambda xs: (ctypes.c_void_p * len(xs))(*xs)
    ok = arr([256, 512])
    # no layers, too many layers, NULL arrays, mismatched head_dim: refused on the host
    assert lib.build_segpaged_cache_layers(0, arr([a]), arr([256]), arr([256]), arr([256]), 0, 0, 64, 256, 256,
                                           None) == S.SP_ERR_INVALID_ARG
    assert lib.build_segpaged_cache_layers(129, arr([a] * 129), arr([256] * 129), arr([256] * 129),
                                           arr([256] * 129), 0, 0, 64, 256, 256, None) == S.SP_ERR_INVALID_ARG
    assert lib.build_segpaged_cache_layers(2, None, ok, ok, ok, 0, 0, 64, 256, 256, None) == S.SP_ERR_INVALID_ARG
    assert lib.build_segpaged_cache_layers(2, arr([a, b]), ok, ok, ok, 0, 0, 64, 256, 256,
                                           None) == S.SP_ERR_INVALID_ARG
    assert "same dtype" in S.last_error()
    S.segpaged_plan_destroy(a)
    S.segpaged_plan_destroy(b)


def test_ring_plan_spare_pool_ids_and_checks():
    """With a shared spare pool, a GLOBAL head's reserved records have no page (-1) and the plan owns
    its assigned pages plus the pool; page_ids permute both; the pool needs a ring plan."""
    L0 = (70, 200, 5)
    pol = [("local", 4, 40), ("global", 0, 0)] * 3
    base = S.make_problem(3, 4, 2, 128, 64, "bf16", L0, [L - 1 for L in L0], pol, flags=S.SP_FLAG_RING,
                          append_capacity=150)
    plan = S.segpaged_plan_create(base)
    z0 = S.segpaged_plan_sizes(plan)
    full = [S.segpaged_plan_head_pages(plan, b, 1) for b in range(3)]
    S.segpaged_plan_destroy(plan)
    spare = 3
    p = S.make_problem(3, 4, 2, 128, 64, "bf16", L0, [L - 1 for L in L0], pol, flags=S.SP_FLAG_RING,
                       append_capacity=150, spare_pages=spare)
    plan = S.segpaged_plan_create(p)
    z = S.segpaged_plan_sizes(plan)
    heads = [S.segpaged_plan_head_pages(plan, b, 1) for b in range(3)]
    local = [S.segpaged_plan_head_pages(plan, b, 0) for b in range(3)]
    S.segpaged_plan_destroy(plan)
    for L, ids, ids_full in zip(L0, heads, full):
        held = -(-L // 64)
        assert len(ids) == len(ids_full) and all(i >= 0 for i in ids[:held]) and all(i == -1 for i in ids[held:])
    reserved = sum(len(f) - -(-L // 64) for L, f in zip(L0, full))
    assert z.num_pages == z0.num_pages - reserved + spare == z.pool_pages
    owned = sorted(i for ids in heads + local for i in ids if i >= 0)
    assert owned == list(range(z.num_pages - spare))  # records first, the pool's pages after them
    perm = list(np.random.default_rng(4).permutation(z.num_pages) + 2)
    p2 = S.make_problem(3, 4, 2, 128, 64, "bf16", L0, [L - 1 for L in L0], pol, flags=S.SP_FLAG_RING,
                        append_capacity=150, spare_pages=spare, page_ids=perm)
    plan = S.segpaged_plan_create(p2)
    got = sorted(i for b in range(3) for kv in range(2) for i in S.segpaged_plan_head_pages(plan, b, kv) if i >= 0)
    assert got == sorted(perm[:z.num_pages - spare]) and S.segpaged_plan_sizes(plan).pool_pages == max(perm) + 1
    S.segpaged_plan_destroy(plan)
    for bad, code in ((dict(spare_pages=-1, flags=S.SP_FLAG_RING), S.SP_ERR_INVALID_ARG),
                      (dict(spare_pages=2), S.SP_ERR_INVALID_ARG)):
        q = S.make_problem(3, 4, 2, 128, 64, "bf16", L0, [L - 1 for L in L0], pol, **bad)
        st, pl = S.segpaged_plan_create_status(q)
        assert st == code and not pl


def test_block_mass_argument_checks():
    """segpaged_block_mass reports every argument error on the host, before any launch."""
    import ctypes

    def prob(**kw):
        base = dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=64, dtype="bf16",
                    ctx_len=[700, 1300], q_start=[699, 1299], policy=[("global", 0, 0)] * 4)
        base.update(kw)
        return S.make_problem(**base)

    n = ctypes.c_size_t()
    for kw, code in ((dict(page_size=16), S.SP_ERR_UNSUPPORTED), (dict(dtype="f32"), S.SP_ERR_UNSUPPORTED),
                     (dict(head_dim=96), S.SP_ERR_UNSUPPORTED),
                     (dict(num_q_heads=34, num_kv_heads=2, policy=[("global", 0, 0)] * 4), S.SP_ERR_UNSUPPORTED),
                     (dict(num_q_heads=7), S.SP_ERR_UNSUPPORTED),
                     (dict(batch=1100, num_q_heads=64, num_kv_heads=64, ctx_len=[64] * 1100, q_start=[63] * 1100,
                           policy=[("global", 0, 0)] * (1100 * 64)), S.SP_ERR_UNSUPPORTED),  # grid limit
                     (dict(batch=2049, ctx_len=[64] * 2049, q_start=[63] * 2049,
                           policy=[("global", 0, 0)] * (2049 * 2)), S.SP_ERR_UNSUPPORTED),  # batch limit
                     (dict(ctx_len=[700, 0]), S.SP_ERR_INVALID_ARG)):
        assert S.load().segpaged_block_mass_workspace(ctypes.byref(prob(**kw)), ctypes.byref(n)) == code, kw
    p = prob()
    ws = S.segpaged_block_mass_workspace(p)
    assert ws == -(-2 * 2 * 8 * 21 * 4 // 256) * 256  # 2 floats per (q-head, block), 21 blocks of the longest
    good = (1 << 20, 128 * 2048 * 2, 2048 * 128, 128, 2 << 20, 0.0, 4 << 20, 21, 8 << 20, ws, None)
    for i, bad, code in ((0, 0, S.SP_ERR_INVALID_ARG), (0, 8, S.SP_ERR_INVALID_ARG),  # NULL, misaligned keys
                         (3, 12, S.SP_ERR_INVALID_ARG),                                 # stride not a multiple of 8
                         (4, 0, S.SP_ERR_INVALID_ARG), (6, 0, S.SP_ERR_INVALID_ARG),    # NULL q, NULL mass
                         (5, float("nan"), S.SP_ERR_INVALID_ARG),                      # scale
                         (7, 20, S.SP_ERR_INVALID_ARG),                                 # mass_stride < 21 blocks
                         (8, 64, S.SP_ERR_INVALID_ARG),                                 # workspace not 256-aligned
                         (9, ws - 256, S.SP_ERR_WORKSPACE)):
        args = list(good)
        args[i] = bad
        assert S.segpaged_block_mass_status(p, *args) == code, (i, bad, S.last_error())


def test_runtime_block_mass_rejects_bad_tensors():
    """runtime.block_mass checks dtypes, shapes and lengths before it reaches the library."""
    import torch

    from head_aware_paged_build_b200.runtime import block_mass

    k = torch.zeros(2, 2, 128, 64, dtype=torch.bfloat16)
    q = torch.zeros(2, 8, 64, dtype=torch.bfloat16)
    for kk, qq, lens in ((k.float(), q, [128, 100]), (k, q.float(), [128, 100]),   # dtypes
                         (k, q[:, :7], [128, 100]),                                 # Hq not a multiple of Hkv
                         (k, q[:, :, :32], [128, 100]),                             # head_dim mismatch
                         (k, q, [129, 100]), (k, q, [0, 100]), (k, q, [128])):      # lengths
        with pytest.raises(ValueError):
            block_mass(kk, qq, lens)
