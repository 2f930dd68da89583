"""Ring plans and in-place decode appends with LOCAL eviction, against the oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _parity import assert_close, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


@pytest.mark.parametrize("dtype,page,d,g", [("f32", 16, 64, 2), ("bf16", 64, 128, 4), ("bf16", 64, 64, 1)])
def test_ring_appends_match_oracle_every_step(dtype, page, d, g):
    """Build at L0, then append N tokens one step at a time; every ring wraps several times.

    After each checked step the decode output (query at the new position) matches the oracle over
    the grown context, and at the end the gathered cache holds exactly the oracle's stored set.
    """
    L0 = (70, 200, 5, 131)
    N = 150 if page == 16 else 140
    pol = []
    for _ in L0:
        pol += [("local", 4, 20 if page == 16 else 40), ("global", 0, 0), ("local", 0, 3 if page == 16 else 64),
                ("local", 300, 10)]
    hkv = 4
    final = tuple(L + N for L in L0)
    wl = W.custom("ring", 61, len(L0), hkv * g, hkv, d, dtype, page, final, pol)
    k, v = W.dense_kv(W.Problem(wl, final, tuple(L - 1 for L in final)), device="cuda")
    qall = W.queries(W.Problem(wl, final, tuple(L - 1 for L in L0)), device="cuda")  # positions L0-1 .. final-1
    qoff = W.Problem(wl, final, tuple(L - 1 for L in L0)).q_offsets
    start = W.Problem(wl, L0, tuple(L - 1 for L in L0))
    layer = layer_for(start, flags=S.SP_FLAG_RING, append_capacity=N)
    layer.build(k, v)
    out = torch.empty(len(L0), hkv * g, d, dtype=k.dtype, device="cuda")
    lse = torch.empty(len(L0), hkv * g, dtype=torch.float32, device="cuda")
    check = set(range(0, N, 9)) | {N - 2, N - 1}
    for i in range(N):
        pos = [L + i for L in L0]
        kn = torch.stack([k[b, :, p] for b, p in enumerate(pos)]).contiguous()
        vn = torch.stack([v[b, :, p] for b, p in enumerate(pos)]).contiguous()
        layer.append(kn, vn)
        q = torch.stack([qall[qoff[b] + 1 + i] for b in range(len(L0))]).contiguous()
        layer.attention(q, out, lse)
        if i in check:
            torch.cuda.synchronize()
            prob = W.Problem(wl, tuple(p + 1 for p in pos), tuple(pos))
            assert_close(compare(prob, q, k, v, out, lse), dtype)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    ko, vo = torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
    layer.gather(ko, vo)
    torch.cuda.synchronize()
    kb, vb, kob, vob = _bits(k.cpu()), _bits(v.cpu()), _bits(ko.cpu()), _bits(vo.cpu())
    sentinel = _bits(torch.full((1,), float("nan"), dtype=k.dtype))[0]
    for b, L in enumerate(final):
        for kv in range(hkv):
            kind, s, w = pol[b * hkv + kv]
            m = torch.from_numpy(oracle.stored_mask(kind, s, w, L, L - 1))
            assert torch.equal(kob[b, kv, :L][m], kb[b, kv, :L][m]), (b, kv)
            assert torch.equal(vob[b, kv, :L][m], vb[b, kv, :L][m]), (b, kv)
            assert bool((kob[b, kv, :L][~m] == sentinel).all()), (b, kv)


def test_ring_append_beyond_capacity_reports_and_skips():
    """A GLOBAL head with no reserved page left: the append is skipped and the status word says so."""
    wl = W.custom("cap", 62, 1, 2, 2, 128, "bf16", 64, (80,), [("global", 0, 0), ("local", 4, 8)])
    prob = W.Problem(wl, (60,), (59,))
    k, v = W.dense_kv(W.Problem(wl, (80,), (79,)), device="cuda")
    layer = layer_for(prob, flags=S.SP_FLAG_RING, append_capacity=0)
    layer.build(k, v)
    for p in range(60, 64):  # the last page still has slots 60..63
        layer.append(k[:, :, p].contiguous(), v[:, :, p].contiguous())
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    layer.append(k[:, :, 64].contiguous(), v[:, :, 64].contiguous())
    torch.cuda.synchronize()
    assert layer.device_status() == 6


@pytest.mark.parametrize("kv_dtype", [None, "e4m3"])
def test_decode_step_graph_matches_eager_steps(kv_dtype):
    """A serving step replayed from a CUDA graph gives bitwise the eager step's O and LSE, step after step."""
    from head_aware_paged_build_b200.runtime import DecodeStepGraph
    L0, N = (300, 77, 130), 40
    pol = [("local", 4, 64), ("global", 0, 0)] * len(L0)
    final = tuple(L + N for L in L0)
    wl = W.custom("graph", 67, len(L0), 8, 2, 128, "bf16", 64, final, pol)
    k, v = W.dense_kv(W.Problem(wl, final, tuple(L - 1 for L in final)), device="cuda")
    qprob = W.Problem(wl, final, tuple(L - 1 for L in L0))
    qall, qoff = W.queries(qprob, device="cuda"), qprob.q_offsets
    kw = dict(kv_dtype="e4m3", k_scale=0.02, v_scale=0.02) if kv_dtype else {}
    start = W.Problem(wl, L0, tuple(L - 1 for L in L0))
    eager = layer_for(start, flags=S.SP_FLAG_RING, append_capacity=N, **kw)
    graphed = layer_for(start, flags=S.SP_FLAG_RING, append_capacity=N, **kw)
    eager.build(k, v)
    graphed.build(k, v)
    step = DecodeStepGraph(graphed)
    out = torch.empty(len(L0), 8, 128, dtype=k.dtype, device="cuda")
    lse = torch.empty(len(L0), 8, dtype=torch.float32, device="cuda")
    for i in range(N):
        pos = [L + i for L in L0]
        kn = torch.stack([k[b, :, p] for b, p in enumerate(pos)]).contiguous()
        vn = torch.stack([v[b, :, p] for b, p in enumerate(pos)]).contiguous()
        q = torch.stack([qall[qoff[b] + 1 + i] for b in range(len(L0))]).contiguous()
        eager.append(kn, vn)
        eager.attention(q, out, lse)
        step.k_in.copy_(kn.cpu()), step.v_in.copy_(vn.cpu()), step.q_in.copy_(q.cpu())
        step.replay()
        torch.cuda.synchronize()
        assert torch.equal(step.out, out.cpu()), i
        assert torch.equal(step.lse, lse.cpu()), i
    assert eager.device_status() == 0 and graphed.device_status() == 0
    if kv_dtype is None:  # and the last step against the oracle
        prob = W.Problem(wl, tuple(p + 1 for p in pos), tuple(pos))
        assert_close(compare(prob, q, k, v, step.out, step.lse), "bf16")
