"""Pins of the CPU oracle against facts fixed outside it (no GPU needed).

Each pin is chosen so that a plausible mistake in the oracle (an off-by-one
window, sinks counted from the chunk, a dropped scale, a transposed operand,
a wrong GQA map) fails at least one of them; ``test_oracle_mutants.py`` plants
such mistakes and checks that they are caught.
"""
from __future__ import annotations

import math
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from head_aware_paged_build_b200 import workloads as W

GOLDEN = Path(__file__).parent / "golden"


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _read_golden(name):
    kv = {}
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = (x.strip() for x in line.split("=", 1))
        kv[k] = v
    return kv


# (kind, sink, window) grid covering window 1, window < sink, overlap, s = 0, w >= L
POLICIES = [("global", 0, 0), ("dense", 0, 0), ("local", 0, 1), ("local", 0, 2), ("local", 1, 1),
            ("local", 4, 8), ("local", 3, 100), ("local", 8, 3), ("local", 2, 5)]


@pytest.mark.parametrize("kind,sink,window", POLICIES)
@pytest.mark.parametrize("L,q0,d", [(1, 0, 4), (9, 0, 8), (23, 11, 8), (40, 39, 16)])
def test_oracle_matches_brute_force(kind, sink, window, L, q0, d):
    rng = np.random.default_rng(1000 * L + 10 * d + sink + 7 * window)
    q, k, v = _rand(rng, L - q0, d), _rand(rng, L, d), _rand(rng, L, d)
    scale = 1.0 / math.sqrt(d)
    pos = np.arange(q0, L)
    out, lse = oracle.attention_rows(q, pos, k, v, kind, sink, window)
    for i, p in enumerate(pos):
        bo, bl = brute.attention_row(q[i].tolist(), k.tolist(), v.tolist(), kind, sink, window, int(p), scale)
        np.testing.assert_allclose(out[i], bo, rtol=0, atol=1e-12)
        assert abs(lse[i] - bl) <= 1e-12


def test_global_head_is_causal_attention():
    """GLOBAL = ordinary causal attention (library SDPA, fp64 CPU, bottom-right mask)."""
    rng = np.random.default_rng(5)
    L, C, d = 70, 30, 32
    q, k, v = _rand(rng, C, d), _rand(rng, L, d), _rand(rng, L, d)
    pos = np.arange(L - C, L)
    out, _ = oracle.attention_rows(q, pos, k, v, "global", 0, 0)
    mask = torch.from_numpy(np.arange(L)[None, :] <= pos[:, None])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None], attn_mask=mask[None])
    np.testing.assert_allclose(out, ref[0].numpy(), rtol=0, atol=1e-12)


def test_local_head_is_sdpa_with_sink_window_mask():
    """LOCAL = SDPA with the sink-plus-window mask written from the text as sets."""
    rng = np.random.default_rng(6)
    L, C, d, s, w = 90, 50, 16, 3, 17
    q, k, v = _rand(rng, C, d), _rand(rng, L, d), _rand(rng, L, d)
    pos = np.arange(L - C, L)
    mask = np.zeros((C, L), bool)
    for i, p in enumerate(pos):
        mask[i, brute.visible_positions("local", s, w, int(p))] = True
    out, _ = oracle.attention_rows(q, pos, k, v, "local", s, w)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=torch.from_numpy(mask)[None])
    np.testing.assert_allclose(out, ref[0].numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("sink", [0, 4])
def test_local_with_window_covering_context_equals_global(sink):
    rng = np.random.default_rng(7)
    L, d = 50, 8
    q, k, v = _rand(rng, L, d), _rand(rng, L, d), _rand(rng, L, d)
    pos = np.arange(L)
    og, lg = oracle.attention_rows(q, pos, k, v, "global", 0, 0)
    ol, ll = oracle.attention_rows(q, pos, k, v, "local", sink, L)
    assert np.array_equal(og, ol) and np.array_equal(lg, ll)


def test_window_one_returns_own_value():
    """sink 0, window 1: each query sees only itself, so O = V[p] and LSE = s_pp."""
    rng = np.random.default_rng(8)
    L, d = 33, 8
    q, k, v = _rand(rng, L, d), _rand(rng, L, d), _rand(rng, L, d)
    pos = np.arange(L)
    out, lse = oracle.attention_rows(q, pos, k, v, "local", 0, 1)
    assert np.array_equal(out, v)
    np.testing.assert_allclose(lse, (q * k).sum(1) / math.sqrt(d), rtol=0, atol=1e-13)


def test_window_two_with_equal_keys_averages_last_two_values():
    rng = np.random.default_rng(9)
    L, d = 20, 8
    q, v = _rand(rng, L, d), _rand(rng, L, d)
    k = np.tile(_rand(rng, 1, d), (L, 1))
    pos = np.arange(1, L)
    out, _ = oracle.attention_rows(q[1:], pos, k, v, "local", 0, 2)
    np.testing.assert_allclose(out, (v[:-1] + v[1:]) / 2, rtol=0, atol=1e-15)


@pytest.mark.parametrize("sink,window", [(4, 8), (0, 5), (6, 1), (3, 3)])
def test_equal_keys_average_visible_values_and_count(sink, window):
    """All keys equal: O is the mean of the visible values, |V(p)| = min(p+1, s+w)."""
    rng = np.random.default_rng(10 + sink)
    L, d = 40, 4
    q = _rand(rng, L, d)
    k = np.tile(_rand(rng, 1, d), (L, 1))
    v = np.zeros((L, d))
    v[:, 0] = 1.0                       # column 0 counts the visible rows via LSE
    v[:, 1] = np.arange(L, dtype=float)  # column 1 gives the mean visible position
    v[:, 2:] = _rand(rng, L, d - 2)
    pos = np.arange(L)
    out, lse = oracle.attention_rows(q, pos, k, v, "local", sink, window)
    for i, p in enumerate(pos):
        n_vis = min(p + 1, sink + window)
        s = float(q[i] @ k[0]) / 2.0
        assert abs(lse[i] - (s + math.log(n_vis))) <= 1e-12
        vis = [j for j in range(p + 1) if j < sink or j > p - window]
        assert len(vis) == n_vis
        np.testing.assert_allclose(out[i, 1], np.mean(vis), rtol=0, atol=1e-12)
        np.testing.assert_allclose(out[i, 2:], v[vis, 2:].mean(0), rtol=0, atol=1e-12)


def test_batched_rows_of_mixed_groups_match_brute_force():
    """The batched call (many groups, each with its own context length and policy) against brute force,
    and bit for bit against one call per group (each row is computed by the same code whichever call runs it)."""
    rng = np.random.default_rng(21)
    d = 8
    groups = []
    for gi, (kind, sink, window) in enumerate(POLICIES):
        L = 5 + 7 * gi
        q0 = max(0, L - 1 - 3 * gi)
        groups.append((_rand(rng, L - q0, d), np.arange(q0, L), _rand(rng, L, d), _rand(rng, L, d), kind, sink,
                       window))
    res = oracle.attention_batch(groups)
    scale = 1.0 / math.sqrt(d)
    for (q, pos, k, v, kind, sink, window), (out, lse) in zip(groups, res):
        for i, p in enumerate(pos):
            bo, bl = brute.attention_row(q[i].tolist(), k.tolist(), v.tolist(), kind, sink, window, int(p), scale)
            np.testing.assert_allclose(out[i], bo, rtol=0, atol=1e-12)
            assert abs(lse[i] - bl) <= 1e-12
        o1, l1 = oracle.attention_rows(q, pos, k, v, kind, sink, window)
        assert np.array_equal(o1, out) and np.array_equal(l1, lse)
    with pytest.raises(ValueError):
        q, pos, k, v, kind, sink, window = groups[0]
        oracle.attention_batch([(q, pos + 100, k, v, kind, sink, window)])


def test_gqa_equals_mha_with_repeated_kv_heads():
    """Query head h uses kv-head h // g: repeating each kv-head g times gives the same result."""
    rng = np.random.default_rng(11)
    L, d, hkv, g = 24, 8, 2, 3
    q = _rand(rng, hkv * g, L, d)
    k, v = _rand(rng, hkv, L, d), _rand(rng, hkv, L, d)
    pol = [("global", 0, 0), ("local", 2, 5)]
    pos = np.arange(L)
    for h in range(hkv * g):
        kv = h // g
        a, _ = oracle.attention_rows(q[h], pos, k[kv], v[kv], *pol[kv])
        k_rep, v_rep = np.repeat(k, g, 0), np.repeat(v, g, 0)
        b, _ = oracle.attention_rows(q[h], pos, k_rep[h], v_rep[h], *pol[h // g])
        assert np.array_equal(a, b)


def test_scale_override_and_positions_outside_context_rejected():
    rng = np.random.default_rng(12)
    L, d = 10, 4
    q, k, v = _rand(rng, 1, d), _rand(rng, L, d), _rand(rng, L, d)
    out, lse = oracle.attention_rows(q, [9], k, v, "global", 0, 0, scale=0.0)
    np.testing.assert_allclose(out[0], v.mean(0), atol=1e-15)
    assert abs(lse[0] - math.log(L)) < 1e-14
    with pytest.raises(ValueError):
        oracle.attention_rows(q, [10], k, v, "global", 0, 0)


@pytest.mark.parametrize("kind,sink,window", POLICIES)
@pytest.mark.parametrize("L,q0", [(1, 0), (17, 16), (30, 0), (64, 40), (5, 3)])
def test_stored_mask_matches_brute_union(kind, sink, window, L, q0):
    m = oracle.stored_mask(kind, sink, window, L, q0)
    keep = brute.stored_positions(kind, sink, window, L, q0)
    assert set(np.flatnonzero(m).tolist()) == keep
    pairs = oracle.visible_pairs(kind, sink, window, L, q0)
    assert pairs == sum(len(brute.visible_positions(kind, sink, window, p)) for p in range(q0, L))


def test_stored_counts_closed_forms_at_decode():
    """Decode keeps L tokens for a global head and min(L, s + w) for a local head."""
    for L in (1, 3, 4, 5, 100, 517, 516, 515, 2000):
        assert oracle.stored_mask("global", 0, 0, L, L - 1).sum() == L
        assert oracle.stored_mask("local", 4, 512, L, L - 1).sum() == min(L, 516)
        m = oracle.stored_mask("local", 4, 512, L, L - 1)
        assert m[: min(4, L)].all() and m[max(0, L - 512):].all()


def test_stored_counts_of_the_synthetic_layers():
    """Closed-form stored token-heads: global L, local min(L, s + w + C - 1) (chunk of C queries)."""
    def closed(wl, prob):
        n = 0
        for b in range(wl.batch):
            L, q0 = prob.ctx_lens[b], prob.q_starts[b]
            for kv in range(wl.num_kv_heads):
                kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
                n += L if kind != "local" else min(L, s + w + (L - q0) - 1)
        return n

    expect = {"tiny": (293, 512), "mistral": (77920, 127048), "llama": (721120, 950440)}
    for name, (dec, pre) in expect.items():
        wl = W.ALL[name]()
        assert closed(wl, wl.decode_problem()) == dec
        assert closed(wl, wl.prefill_problem()) == pre
    # brute-force union on the tiny layer agrees with the closed form
    wl = W.tiny()
    for prob, want in ((wl.decode_problem(), 293), (wl.prefill_problem(), 512)):
        got = sum(oracle.stored_mask(*wl.policy[kv], prob.ctx_lens[0], prob.q_starts[0]).sum()
                  for kv in range(2))
        assert got == want
    assert closed(W.mha(), W.mha().decode_problem()) == 4 * (8 * 131072 + 56 * 132)


def test_visible_flops_of_tiny_prefill():
    """Visible pairs of the tiny prefill: 2 q-heads x (global 256*257/2 + local sum_p min(p+1, 36))."""
    wl = W.tiny()
    glob = 256 * 257 // 2
    loc = sum(min(p + 1, 36) for p in range(256))
    got = 2 * (oracle.visible_pairs("global", 0, 0, 256, 0) + oracle.visible_pairs("local", 4, 32, 256, 0))
    assert got == 2 * (glob + loc)
    assert 4 * wl.head_dim * got == 21_238_784  # 2.12e7 visible FLOPs


def test_golden_deepseek_policy_savings():
    """The page's DeepSeek-V4-Flash policy: 56 of 64 heads local (87.5%), window 128, sink 4."""
    g = _read_golden("deepseek_v4_flash_policy.txt")
    n = int(g["heads_per_layer"])
    glob = {int(x) for x in g["global_head_ids"].split(",")}
    s, w = int(g["local_sink"]), int(g["local_window"])
    assert glob == set(range(0, n, 8))
    frac_local = (n - len(glob)) / n
    assert frac_local == float(g["local_head_fraction_middle"])
    for L in (65536, 131072, 262144):
        stored = sum(int(oracle.stored_mask("global" if h in glob else "local", s, w, L, L - 1).sum())
                     for h in range(n))
        saving = 1 - stored / (n * L)
        assert saving == pytest.approx(frac_local * (1 - (s + w) / L), abs=1e-12)
        assert float(g["kv_saving_low"]) <= saving <= float(g["kv_saving_high"])
    assert int(g["default_window"]) == 512 and int(g["default_sink"]) == 4


def test_e4m3_codes_fixed_by_the_format():
    """Values fixed by the E4M3 definition (bias 7, 3 mantissa bits, max 448, subnormal step 2^-9)."""
    vals = np.array([0.0, 1.0, -1.0, 448.0, 500.0, -1e6, 2.0 ** -9, 2.0 ** -6, 1.125, 0.875 * 2 ** -6,
                     240.0, 256.0], np.float32)
    want = [0x00, 0x38, 0xB8, 0x7E, 0x7E, 0xFE, 0x01, 0x08, 0x39, 0x07, 0x77, 0x78]
    assert oracle.e4m3_encode(vals, 1.0).tolist() == want
    back = oracle.e4m3_decode(np.array(want, np.uint8), 1.0)
    np.testing.assert_array_equal(back, [0, 1, -1, 448, 448, -448, 2 ** -9, 2 ** -6, 1.125, 0.875 * 2 ** -6, 240, 256])
    # a decoded value is the code's value times the scale: 1.0 (0x38) at scale 0.25, -448 (0xFE) at 2
    np.testing.assert_array_equal(oracle.e4m3_decode(np.array([0x38, 0xFE], np.uint8), 0.25), [0.25, -112.0])


def test_e4m3_rounds_to_nearest_even_and_saturates():
    # 1.0625 lies halfway between 1.0 (code 0x38, even) and 1.125 (0x39): ties to even -> 1.0
    # 1.1875 lies halfway between 1.125 (0x39) and 1.25 (0x3A, even) -> 1.25
    assert oracle.e4m3_encode(np.array([1.0625, 1.1875, 1.07], np.float32), 1.0).tolist() == [0x38, 0x3A, 0x39]
    # every code's value encodes back to itself; scaling divides by the scale before rounding
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = oracle.e4m3_decode(codes, 1.0).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals, 1.0)[codes != 0x80], codes[codes != 0x80])
    assert oracle.e4m3_encode(np.array([3.0], np.float32), 0.5).tolist() == [0x3C]  # 1.5 -> 0.0111.100
    # brute force: the chosen code is a nearest finite value of every random input
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(2000) * 50).astype(np.float32)
    c = oracle.e4m3_encode(x, 1.0)
    finite = oracle.e4m3_decode(codes, 1.0)
    best = np.abs(x[:, None].astype(np.float64) - finite[None, :]).min(1)
    got = np.abs(x.astype(np.float64) - oracle.e4m3_decode(c, 1.0))
    clipped = np.abs(x) > 448
    assert np.all(got[~clipped] == best[~clipped])


def test_e4m3_every_midpoint_goes_to_the_even_neighbour():
    """Halfway between any two adjacent finite values (exact in fp32) the even code wins, both signs."""
    codes = np.arange(0x7F, dtype=np.uint8)  # 0 .. 0x7E: increasing values
    vals = oracle.e4m3_decode(codes, 1.0)
    mid = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (vals[:-1] + vals[1:]) / 2)  # exact in fp32
    even = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[1:])
    assert np.array_equal(oracle.e4m3_encode(mid, 1.0), even)
    assert np.array_equal(oracle.e4m3_encode(-mid, 1.0), even | 0x80)
    # just above / below each midpoint: the nearer neighbour
    up = np.nextafter(mid, np.float32(np.inf))
    down = np.nextafter(mid, np.float32(0))
    assert np.array_equal(oracle.e4m3_encode(up, 1.0), codes[1:])
    assert np.array_equal(oracle.e4m3_encode(down, 1.0), codes[:-1])
    # the subnormal range against brute force
    x = np.random.default_rng(5).uniform(-2.0 ** -5, 2.0 ** -5, 4000).astype(np.float32)
    c = oracle.e4m3_encode(x, 1.0)
    best = np.abs(x[:, None].astype(np.float64) - np.concatenate([vals, -vals])[None, :]).min(1)
    assert np.all(np.abs(x.astype(np.float64) - oracle.e4m3_decode(c, 1.0)) == best)


# ---------------------------------------------------------------------------
# RETRIEVAL heads: sink + recent window + the top-p blocks by importance
# ---------------------------------------------------------------------------

def _masses(rng, n, integer):
    return (rng.integers(0, 6, n) if integer else rng.exponential(1.0, n)).astype(np.float32)


@pytest.mark.parametrize("integer", [True, False])
@pytest.mark.parametrize("top_p", [0.0, 0.25, 0.5, 0.7, 0.9, 1.0])
@pytest.mark.parametrize("L,block,sink", [(1, 4, 0), (13, 4, 0), (29, 4, 3), (32, 8, 8), (40, 8, 11), (37, 16, 0)])
def test_retrieval_selection_matches_exhaustive_search(integer, top_p, L, block, sink):
    """The kept blocks are the fewest whose importance reaches top_p of the total (exhaustive search)."""
    rng = np.random.default_rng(hash((integer, top_p, L, block, sink)) % (1 << 32))
    n = -(-L // block)
    for _ in range(4):
        mass = _masses(rng, n, integer)
        sel = oracle.retrieval_select(L, block, sink, top_p, mass)
        want = brute.kept_blocks(L, block, sink, float(np.float32(top_p)), [float(x) for x in mass])
        assert set(np.flatnonzero(sel).tolist()) == want, (mass, top_p)


def test_retrieval_selection_closed_forms():
    """Uniform importance keeps ceil(top_p * candidates) blocks, lowest first; a single heavy block is kept alone."""
    for n_cand, top_p in [(10, 0.25), (10, 0.5), (7, 0.75), (16, 0.5), (5, 1.0), (5, 0.0)]:
        L, block, sink = 64 * (n_cand + 1), 64, 64  # block 0 is all sink: not a candidate
        sel = oracle.retrieval_select(L, block, sink, top_p, np.ones(n_cand + 1, np.float32))
        k = math.ceil(top_p * n_cand)
        assert not sel[0] and sel.sum() == k and np.array_equal(np.flatnonzero(sel), np.arange(1, k + 1))
    mass = np.zeros(9, np.float32)
    mass[6] = 3.5
    for top_p in (0.01, 0.5, 0.99):
        assert np.flatnonzero(oracle.retrieval_select(9 * 32, 32, 4, top_p, mass)).tolist() == [6]
    with pytest.raises(ValueError):
        oracle.retrieval_select(64, 32, 0, 0.5, np.array([1.0, -1.0], np.float32))
    with pytest.raises(ValueError):
        oracle.retrieval_select(64, 32, 0, 0.5, np.array([1.0, np.inf], np.float32))


@pytest.mark.parametrize("top_p", [0.3, 0.6, 0.95])
@pytest.mark.parametrize("sink,window", [(0, 1), (2, 3), (4, 8), (9, 2)])
@pytest.mark.parametrize("L,q0,block", [(17, 0, 4), (33, 20, 4), (40, 39, 8), (29, 10, 8)])
def test_retrieval_attention_matches_brute_force(top_p, sink, window, L, q0, block):
    rng = np.random.default_rng(L * 1000 + q0 * 10 + sink + window)
    d = 8
    q, k, v = _rand(rng, L - q0, d), _rand(rng, L, d), _rand(rng, L, d)
    mass = _masses(rng, -(-L // block), False)
    sel = oracle.retrieval_select(L, block, sink, top_p, mass)
    kept = set(np.flatnonzero(sel).tolist())
    pos = np.arange(q0, L)
    out, lse = oracle.attention_rows(q, pos, k, v, "retrieval", sink, window, sel=sel, block=block)
    scale = 1.0 / math.sqrt(d)
    for i, p in enumerate(pos):
        bo, bl = brute.attention_row(q[i].tolist(), k.tolist(), v.tolist(), "retrieval", sink, window, int(p), scale,
                                     kept, block)
        np.testing.assert_allclose(out[i], bo, rtol=0, atol=1e-12)
        assert abs(lse[i] - bl) <= 1e-12
    # the stored set is the union of the rows' visible sets, the pair count their sizes
    stored = oracle.stored_mask("retrieval", sink, window, L, q0, sel=sel, block=block)
    assert set(np.flatnonzero(stored).tolist()) == brute.stored_positions("retrieval", sink, window, L, q0, kept,
                                                                          block)
    pairs = sum(len(brute.visible_positions("retrieval", sink, window, int(p), kept, block)) for p in pos)
    assert oracle.visible_pairs("retrieval", sink, window, L, q0, sel=sel, block=block) == pairs


@pytest.mark.parametrize("sink,window", [(0, 1), (4, 8), (3, 100)])
def test_retrieval_top_p_one_is_global_and_zero_is_local(sink, window):
    rng = np.random.default_rng(31 + sink)
    L, d, block, q0 = 70, 16, 8, 30
    q, k, v = _rand(rng, L - q0, d), _rand(rng, L, d), _rand(rng, L, d)
    mass = _masses(rng, -(-L // block), False)
    mass[3] = 0.0  # a zero-importance block is still kept at top_p = 1
    pos = np.arange(q0, L)
    s1 = oracle.retrieval_select(L, block, sink, 1.0, mass)
    o1, l1 = oracle.attention_rows(q, pos, k, v, "retrieval", sink, window, sel=s1, block=block)
    og, lg = oracle.attention_rows(q, pos, k, v, "global", 0, 0)
    assert np.array_equal(o1, og) and np.array_equal(l1, lg)
    s0 = oracle.retrieval_select(L, block, sink, 0.0, mass)
    assert not s0.any()
    o0, l0 = oracle.attention_rows(q, pos, k, v, "retrieval", sink, window, sel=s0, block=block)
    ol, ll = oracle.attention_rows(q, pos, k, v, "local", sink, window)
    assert np.array_equal(o0, ol) and np.array_equal(l0, ll)


def test_retrieval_equal_keys_average_the_kept_values():
    """All keys equal: every visible weight is the same, so O is the mean of the visible values and
    |V(p)| = (kept or sink positions before the window) + (window positions up to p)."""
    rng = np.random.default_rng(44)
    L, d, block, sink, window = 48, 4, 8, 2, 5
    k = np.tile(_rand(rng, 1, d), (L, 1))
    v = _rand(rng, L, d)
    q = _rand(rng, L, d)
    mass = np.array([0, 9, 0, 4, 0, 1], np.float32)
    sel = oracle.retrieval_select(L, block, sink, 0.9, mass)
    assert np.flatnonzero(sel).tolist() == [1, 3]  # 9 + 4 = 13 >= 0.9 * 14
    out, lse = oracle.attention_rows(q, np.arange(L), k, v, "retrieval", sink, window, sel=sel, block=block)
    for p in range(L):
        lo = max(0, p - window + 1)
        early = [j for j in range(lo) if j < sink or sel[j // block]]
        vis = early + list(range(lo, p + 1))
        np.testing.assert_allclose(out[p], v[vis].mean(0), rtol=0, atol=1e-12)
        s0 = float(q[p] @ k[0]) / math.sqrt(d)
        assert abs(lse[p] - (s0 + math.log(len(vis)))) < 1e-12


# --------------------------------------------------------------------------
# Attention mass per block (the scoring pass behind a retrieval head's importance)
# --------------------------------------------------------------------------

def _mass_by_hand(q, k, block, scale):
    """The definition with Python floats: each query's softmax over all positions, summed per block,
    averaged over the queries."""
    g, L = len(q), len(k)
    nb = -(-L // block)
    out = [0.0] * nb
    for h in range(g):
        s = [scale * math.fsum(a * b for a, b in zip(q[h], k[j])) for j in range(L)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = math.fsum(e)
        for i in range(nb):
            out[i] += math.fsum(e[i * block:(i + 1) * block]) / z / g
    return out


@pytest.mark.parametrize("g,d,L,block", [(1, 4, 9, 4), (2, 8, 37, 8), (4, 16, 64, 16), (3, 5, 1, 4)])
def test_block_mass_matches_brute_force(g, d, L, block):
    rng = np.random.default_rng(g * 100 + L)
    q, k = _rand(rng, g, d), _rand(rng, L, d)
    scale = 1.0 / math.sqrt(d)
    got = oracle.block_mass(q, k, block)
    ref = _mass_by_hand(q.tolist(), k.tolist(), block, scale)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)


def test_block_mass_is_a_distribution():
    rng = np.random.default_rng(5)
    for L, block in ((1000, 64), (999, 64), (65, 64), (64, 64)):
        m = oracle.block_mass(_rand(rng, 8, 32), 3.0 * _rand(rng, L, 32), block)
        assert len(m) == -(-L // block) and (m >= 0).all() and abs(m.sum() - 1.0) < 1e-12


def test_block_mass_equal_keys_is_proportional_to_block_length():
    """Equal keys give every position the same weight: block i's mass is its length over L
    (the ragged last block included)."""
    rng = np.random.default_rng(6)
    L, block = 200, 64
    k = np.tile(_rand(rng, 1, 16), (L, 1))
    m = oracle.block_mass(_rand(rng, 4, 16), k, block)
    lens = np.array([min(block, L - i * block) for i in range(-(-L // block))], np.float64)
    assert np.allclose(m, lens / L, rtol=0, atol=1e-14)


def test_block_mass_dominant_key_and_group_average():
    """One key aligned with the query at 40 sigma takes essentially all of that query's mass; a second
    query of the group that attends uniformly (zero query) spreads its half evenly."""
    rng = np.random.default_rng(7)
    L, d, block = 300, 16, 64
    k = 0.1 * _rand(rng, L, d)
    q0 = _rand(rng, d)
    k[170] = 40.0 * math.sqrt(d) * q0 / (q0 @ q0)  # q0 . k_170 * scale = 40
    m1 = oracle.block_mass(q0[None], k, block)
    assert m1[170 // block] > 1 - 1e-12
    m2 = oracle.block_mass(np.stack([q0, np.zeros(d)]), k, block)  # the zero query weighs every key 1 / L
    lens = np.array([min(block, L - i * block) for i in range(-(-L // block))], np.float64)
    assert np.allclose(m2, (m1 + lens / L) / 2, rtol=0, atol=1e-14)
