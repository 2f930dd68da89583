"""segpaged_decode_step: the append and the decode attention of a serving step in one launch.

Two ring-plan layers start from the same cache; one takes every step through
segpaged_decode_step, the other through segpaged_decode_append followed by
segpaged_attention.  Every step's output and LSE, and at the end the pools and
the device tables, must be equal bit for bit (bf16 and E4M3 pages, LOCAL
rings that wrap many times, windows narrower than a page, heads split over
many CTAs; fp32 plans run the two calls inside the entry point).  A ring
without room reports device code 6 in both, with the same outputs.  A few
steps are also checked against the oracle.
"""
from __future__ import annotations

import pytest
import torch

from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import DecodeStepGraph, layer_for
from _parity import assert_close, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


def _twins(dtype, page, d, g, N, target_ctas=0, kv_dtype=None, capacity=None, L0=(70, 200, 5, 131, 1000)):
    pol = []
    for _ in L0:
        pol += [("local", 4, 20 if page == 16 else 40), ("global", 0, 0), ("local", 0, 3 if page == 16 else 64),
                ("local", 300, 10), ("local", 4, 130)]
    hkv = 5
    final = tuple(L + N for L in L0)
    wl = W.custom("step", 71, len(L0), hkv * g, hkv, d, dtype, page, final, pol)
    k, v = W.dense_kv(W.Problem(wl, final, tuple(L - 1 for L in final)), device="cuda")
    full = W.Problem(wl, final, tuple(L - 1 for L in L0))
    qall, qoff = W.queries(full, device="cuda"), full.q_offsets
    start = W.Problem(wl, L0, tuple(L - 1 for L in L0))
    kw = dict(flags=S.SP_FLAG_RING, append_capacity=N if capacity is None else capacity, target_ctas=target_ctas)
    if kv_dtype:
        kw.update(kv_dtype=kv_dtype, k_scale=float(k.float().abs().max()) / 448,
                  v_scale=float(v.float().abs().max()) / 448)
    a, b = layer_for(start, **kw), layer_for(start, **kw)
    a.build(k, v)
    b.build(k, v)
    return wl, L0, k, v, qall, qoff, a, b


@pytest.mark.parametrize("dtype,page,d,g,ctas,kv_dtype", [
    ("bf16", 64, 128, 4, 0, None), ("bf16", 64, 64, 1, 0, None), ("bf16", 64, 128, 8, 1000, None),
    ("bf16", 64, 128, 4, 0, "e4m3"), ("bf16", 64, 128, 2, 7, "e4m3"), ("f32", 16, 64, 2, 0, None)])
def test_decode_step_equals_append_then_attention(dtype, page, d, g, ctas, kv_dtype):
    N = 150
    wl, L0, k, v, qall, qoff, a, b = _twins(dtype, page, d, g, N, ctas, kv_dtype)
    B, hq = len(L0), wl.num_q_heads
    for i in range(N):
        pos = [L + i for L in L0]
        kn = torch.stack([k[s, :, p] for s, p in enumerate(pos)]).contiguous()
        vn = torch.stack([v[s, :, p] for s, p in enumerate(pos)]).contiguous()
        q = torch.stack([qall[qoff[s] + 1 + i] for s in range(B)]).contiguous()
        oa, la = a.decode_step(kn, vn, q)
        b.append(kn, vn)
        ob, lb = b.attention(q)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob) and torch.equal(la, lb), i
        if kv_dtype is None and i in (0, 77, N - 1):
            prob = W.Problem(wl, tuple(p + 1 for p in pos), tuple(pos))
            assert_close(compare(prob, q, k, v, oa, la), dtype)
    assert a.device_status() == 0 and b.device_status() == 0
    assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool)
    assert torch.equal(a.table, b.table)


def test_decode_step_ring_without_room_reports_like_the_append():
    """Sequence 0 starts at 61 tokens with room for 3 more: its global head's single page is full at
    the 4th step, which both paths skip with device code 6."""
    N = 5
    wl, L0, k, v, qall, qoff, a, b = _twins("bf16", 64, 128, 2, N, capacity=3, L0=(61, 200, 5, 131, 1000))
    B = len(L0)
    for i in range(N):
        pos = [L + i for L in L0]
        kn = torch.stack([k[s, :, p] for s, p in enumerate(pos)]).contiguous()
        vn = torch.stack([v[s, :, p] for s, p in enumerate(pos)]).contiguous()
        q = torch.stack([qall[qoff[s] + 1 + i] for s in range(B)]).contiguous()
        oa, la = a.decode_step(kn, vn, q)
        b.append(kn, vn)
        ob, lb = b.attention(q)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob) and torch.equal(la, lb), i
    assert a.device_status() == 6 and b.device_status() == 6
    assert torch.equal(a.table, b.table) and torch.equal(a.k_pool, b.k_pool)


@pytest.mark.parametrize("kv_dtype", [None, "e4m3"])
def test_decode_step_graph_fused_equals_unfused(kv_dtype):
    """The serving step captured in a CUDA graph, fused and unfused, on the 32K layer at the bench's
    batch of 8 (bf16 and E4M3 pages): outputs every step, and pools and tables at the end, bit for bit."""
    wl = W.llama()
    n = 6
    dec = wl.decode_problem()
    start = W.Problem(wl, tuple(L - n for L in dec.ctx_lens), tuple(L - n - 1 for L in dec.ctx_lens))
    k, v = W.dense_kv(dec, device="cuda", gen_device="cuda")
    kw = {}
    if kv_dtype:
        kw = dict(kv_dtype=kv_dtype, k_scale=float(k.float().abs().max()) / 448,
                  v_scale=float(v.float().abs().max()) / 448)
    steps, layers = [], []
    for fused in (True, False):
        layer = layer_for(start, flags=S.SP_FLAG_RING, append_capacity=n, **kw)
        layer.build(k, v)
        g = DecodeStepGraph(layer, fused=fused)
        outs = []
        for i in range(n):
            pos = [L + i for L in start.ctx_lens]
            g.k_in.copy_(torch.stack([k[b, :, p] for b, p in enumerate(pos)]).cpu())
            g.v_in.copy_(torch.stack([v[b, :, p] for b, p in enumerate(pos)]).cpu())
            g.q_in.copy_(W.queries(W.Problem(wl, tuple(p + 1 for p in pos), tuple(pos)), gen_device="cuda").cpu())
            g.replay()
            torch.cuda.synchronize()
            outs.append((g.out.clone(), g.lse.clone()))
        assert layer.device_status() == 0
        del g
        steps.append(outs)
        layers.append(layer)
    for (oa, la), (ob, lb) in zip(*steps):
        assert torch.equal(oa, ob) and torch.equal(la, lb)
    a, b = layers
    assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool)
    assert torch.equal(a.table, b.table)
