"""Prefill attention against the fp64 oracle, plus invariants."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _parity import assert_close, compare, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


def run_prefill(prob, flags=0, k=None, v=None, q=None, **kw):
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


@pytest.mark.parametrize("flags", [0, S.SP_FLAG_DENSE_MASKED])
def test_tiny_prefill_f32_matches_oracle(flags):
    prob = W.tiny().prefill_problem()
    _, (k, v, q), out, lse = run_prefill(prob, flags=flags)
    assert_close(compare(prob, q, k, v, out, lse), "f32")


@pytest.mark.parametrize("dtype,page,d", [("f32", 16, 64), ("f32", 64, 128), ("bf16", 64, 64), ("bf16", 64, 128)])
@pytest.mark.parametrize("flags", [0, S.SP_FLAG_DENSE_MASKED])
def test_prefill_edge_shapes(dtype, page, d, flags):
    """Ragged chunks (1..300 queries), partial tiles, sink >= L, s = 0 / w = 1, w wider than the context."""
    lens = (1, 2, 63, 129, 200, 300)
    pol = []
    for _ in lens:
        pol += [("global", 0, 0), ("local", 4, 1), ("local", 0, 7), ("local", 70, 3), ("local", 3, 1000),
                ("local", 4, 130)]
    wl = W.custom("edge", 31, len(lens), 12, 6, d, dtype, page, lens, pol, chunk=140)
    prob = wl.prefill_problem()
    _, (k, v, q), out, lse = run_prefill(prob, flags=flags)
    assert_close(compare(prob, q, k, v, out, lse), dtype)


def test_prefill_row_equals_decode_at_same_position():
    """Prefill row p equals a decode query at p over the same tokens and policy (tolerance)."""
    wl = W.custom("pd", 41, 1, 8, 2, 128, "bf16", 64, (700,), [("global", 0, 0), ("local", 4, 100)], chunk=300)
    prob = wl.prefill_problem()
    _, (k, v, q), out, lse = run_prefill(prob)
    for p in (400, 401, 527, 699):
        dec = W.Problem(wl, (p + 1,), (p,))
        layer = layer_for(dec)
        layer.build(k[:, :, : p + 1].contiguous().cuda(), v[:, :, : p + 1].contiguous().cuda())
        o, l = layer.attention(q[p - 400: p - 399].contiguous().cuda())
        torch.cuda.synchronize()
        assert float((o.float() - out[p - 400: p - 399].float()).abs().max()) <= 2e-2
        assert float((l - lse[p - 400: p - 399]).abs().max()) <= 2e-3


@pytest.mark.parametrize("name", ["mistral"])
def test_prefill_bf16_matches_oracle_full(name):
    wl = W.ALL[name]()
    prob = wl.prefill_problem()
    _, (k, v, q), out, lse = run_prefill(prob)
    rows = [sample_rows(c, n_random=64, seed=b) for b, c in enumerate(prob.q_counts)]
    assert_close(compare(prob, q, k, v, out, lse, rows_per_seq=rows), "bf16")


def test_prefill_bf16_page_permutation_and_determinism():
    wl = W.custom("perm", 42, 2, 8, 2, 128, "bf16", 64, (1000, 777), [("global", 0, 0), ("local", 4, 200)] * 2,
                  chunk=400)
    prob = wl.prefill_problem()
    layer, (k, v, q), out0, lse0 = run_prefill(prob)
    out1, lse1 = layer.attention(q.cuda())
    torch.cuda.synchronize()
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)
    n = layer.sizes.num_pages
    perm = list(np.random.default_rng(2).permutation(n))
    _, _, out2, lse2 = run_prefill(prob, k=k, v=v, q=q, page_ids=perm, first_page=1)
    assert torch.equal(out0, out2) and torch.equal(lse0, lse2)


@pytest.mark.parametrize("name", ["llama", "mha"])
def test_prefill_bf16_matches_oracle_sampled_at_full_size(name):
    """The bench's layer (and the MHA 128K layer) at full size, in the bench's launch configuration.

    Inputs are generated on the GPU.  Every sequence and every q-head is checked on chunk
    edges, rows at multiples of 512 and one either side, and seeded random rows; for one
    q-head of a global kv-head and one of a local kv-head of every sequence, also every
    128-row query-tile edge and the rows either side of it.
    """
    wl = W.ALL[name]()
    prob = wl.prefill_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    layer = layer_for(prob)
    layer.build(k, v)
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    rows = [sample_rows(c, stride=512, n_random=12, seed=b) for b, c in enumerate(prob.q_counts)]
    assert_close(compare(prob, q, k, v, out, lse, rows_per_seq=rows), "bf16")
    for b, c in enumerate(prob.q_counts):
        pol = wl.policy[b * wl.num_kv_heads:(b + 1) * wl.num_kv_heads]
        g_kv = next(kv for kv, p in enumerate(pol) if p[0] == "global")
        l_kv = next(kv for kv, p in enumerate(pol) if p[0] == "local")
        edges = [sample_rows(c, stride=128, n_random=4, seed=100 + b) if bb == b else []
                 for bb in range(wl.batch)]
        heads = (g_kv * wl.group, l_kv * wl.group + wl.group - 1)
        assert_close(compare(prob, q, k, v, out, lse, rows_per_seq=edges, heads=heads, seqs=(b,)), "bf16")


def test_prefill_bf16_dense_masked_matches_oracle_at_mistral_size():
    """The dense-plus-mask variant of the bf16 prefill (every head stores its whole context, local heads
    masked per element over every causal tile) on the Mistral-shaped layer, every sequence and q-head."""
    wl = W.mistral()
    prob = wl.prefill_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    layer = layer_for(prob, flags=S.SP_FLAG_DENSE_MASKED)
    layer.build(k, v)
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    rows = [sample_rows(c, stride=128, n_random=16, seed=b) for b, c in enumerate(prob.q_counts)]
    assert_close(compare(prob, q, k, v, out, lse, rows_per_seq=rows), "bf16")


def test_prefill_adaptive_window_matches_oracle():
    lens = (300, 1000, 777)
    pol = []
    for _ in lens:
        pol += [("local", 4, -2), ("global", 0, 0)]
    wl = W.custom("adaptive_p", 52, len(lens), 4, 2, 128, "bf16", 64, lens, pol, chunk=200)
    prob = wl.prefill_problem()
    _, (k, v, q), out, lse = run_prefill(prob)
    resolved = []
    for b, L in enumerate(lens):
        for kind, s, w in pol[2 * b: 2 * b + 2]:
            resolved.append((kind, s, max(1, L // -w) if w < 0 else w))
    ref = W.custom("adaptive_p", 52, len(lens), 4, 2, 128, "bf16", 64, lens, resolved, chunk=200)
    assert_close(compare(ref.prefill_problem(), q, k, v, out, lse), "bf16")
