"""Decode attention (split-KV + combine) against the fp64 oracle, plus invariants."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _parity import assert_close, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


def run_decode(prob, flags=0, k=None, v=None, q=None, **kw):
    if k is None:
        k, v = W.dense_kv(prob)
    if q is None:
        q = W.queries(prob)
    layer = layer_for(prob, flags=flags, **kw)
    layer.build(k.cuda(), v.cuda())
    out, lse = layer.attention(q.cuda())
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return layer, (k, v, q), out, lse


@pytest.mark.parametrize("name", ["tiny", "mistral", "llama", "ragged"])
def test_decode_matches_oracle(name):
    wl = W.ALL[name]()
    prob = wl.decode_problem()
    _, (k, v, q), out, lse = run_decode(prob)
    res = compare(prob, q, k, v, out, lse)
    assert_close(res, wl.dtype)


@pytest.mark.parametrize("name", ["tiny", "mistral"])
def test_decode_dense_masked_variant_matches_oracle(name):
    wl = W.ALL[name]()
    prob = wl.decode_problem()
    _, (k, v, q), out, lse = run_decode(prob, flags=S.SP_FLAG_DENSE_MASKED)
    assert_close(compare(prob, q, k, v, out, lse), wl.dtype)


def test_decode_page_permutation_is_bitwise_invariant():
    prob = W.mistral().decode_problem()
    layer, inputs, out0, lse0 = run_decode(prob)
    n = layer.sizes.num_pages
    perm = list(np.random.default_rng(5).permutation(n))
    _, _, out1, lse1 = run_decode(prob, *(), k=inputs[0], v=inputs[1], q=inputs[2], page_ids=perm, first_page=2)
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)


def test_decode_is_deterministic_and_split_count_invariant():
    prob = W.mistral().decode_problem()
    layer, (k, v, q), out0, lse0 = run_decode(prob)
    out1, lse1 = layer.attention(q.cuda())
    torch.cuda.synchronize()
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)
    for ctas in (1, 7, 150, 400, 1000):  # one item per head up to ~100-slot heads (two-level merges)
        _, _, o, l = run_decode(prob, k=k, v=v, q=q, target_ctas=ctas)
        assert_close(compare(prob, q, k, v, o, l), "bf16")
        assert float((o.float() - out0.float()).abs().max()) <= 2e-2


@pytest.mark.parametrize("dtype,page,d,g", [("f32", 16, 64, 3), ("f32", 64, 128, 16), ("bf16", 64, 64, 1),
                                            ("bf16", 64, 128, 16), ("bf16", 64, 128, 5)])
def test_decode_edge_shapes(dtype, page, d, g):
    """Ragged lengths 1..300, partial pages, sink >= L, s = 0 / w = 1, group sizes 1..16."""
    lens = (1, 2, 63, 64, 65, 129, 300)
    pol = []
    for _ in lens:
        pol += [("global", 0, 0), ("local", 4, 1), ("local", 0, 7), ("local", 70, 3), ("dense", 0, 0)]
    wl = W.custom("edge", 21, len(lens), 5 * g, 5, d, dtype, page, lens, pol)
    prob = wl.decode_problem()
    _, (k, v, q), out, lse = run_decode(prob)
    assert_close(compare(prob, q, k, v, out, lse), dtype)
    _, _, out2, lse2 = run_decode(prob, k=k, v=v, q=q, flags=S.SP_FLAG_DENSE_MASKED)
    assert_close(compare(prob, q, k, v, out2, lse2), dtype)


def test_decode_window_one_returns_own_value():
    """sink 0, window 1: the output is V at the query's own position, rounded to bf16 exactly."""
    wl = W.custom("w1", 22, 2, 8, 2, 128, "bf16", 64, (500, 77), [("local", 0, 1)] * 4)
    prob = wl.decode_problem()
    _, (k, v, q), out, lse = run_decode(prob)
    for b, L in enumerate(prob.ctx_lens):
        for h in range(8):
            assert torch.equal(out[b, h].cpu(), v[b, h // 4, L - 1])


def test_decode_custom_scale():
    wl = W.mistral()
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob)
    q = W.queries(prob)
    layer = layer_for(prob)
    layer.build(k.cuda(), v.cuda())
    out, lse = layer.attention(q.cuda(), scale=0.05)
    torch.cuda.synchronize()
    import oracle
    for b in (0, 3):
        for h in (0, 31):
            kv = h // 4
            kind, s, w = wl.policy[b * 8 + kv]
            o_ref, l_ref = oracle.attention_rows(q[b:b + 1, h].double().numpy(), [8191],
                                                 k[b, kv].double().numpy(), v[b, kv].double().numpy(),
                                                 kind, s, w, scale=0.05)
            assert np.max(np.abs(out[b, h].float().cpu().numpy() - o_ref[0])) <= 2e-2
            assert abs(float(lse[b, h]) - l_ref[0]) <= 2e-3


def test_decode_mha_128k_full_size():
    """MHA 128K layer (64 heads, 8 global, window 128): every output row against the oracle."""
    wl = W.mha()
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    layer = layer_for(prob)
    layer.build(k, v)
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert_close(compare(prob, q, k, v, out, lse), "bf16")


def test_decode_adaptive_window_matches_oracle():
    """Adaptive windows (window = ctx_len // 2 and // 5) against the oracle with the resolved windows."""
    lens = (300, 1000, 2500, 77)
    pol = []
    for _ in lens:
        pol += [("local", 4, -2), ("global", 0, 0), ("local", 0, -5), ("local", 4, 100)]
    wl = W.custom("adaptive", 51, len(lens), 16, 4, 128, "bf16", 64, lens, pol)
    prob = wl.decode_problem()
    _, (k, v, q), out, lse = run_decode(prob)
    resolved = []
    for b, L in enumerate(lens):
        for kind, s, w in pol[4 * b: 4 * b + 4]:
            resolved.append((kind, s, max(1, L // -w) if w < 0 else w))
    ref = W.custom("adaptive", 51, len(lens), 16, 4, 128, "bf16", 64, lens, resolved)
    assert_close(compare(ref.decode_problem(), q, k, v, out, lse), "bf16")
