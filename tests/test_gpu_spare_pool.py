"""Ring plans with a shared spare pool: GLOBAL heads grow into pages taken from one pool.

The GLOBAL heads reserve page records for 150 more tokens but no pages; every
append that reaches a new record takes a page from the plan's spare pool.  With
a pool sized for the batch's growth together, 150 steps match the oracle at
checkpoints, the gathered cache holds exactly the oracle's stored sets, and
the fused decode step gives the same bits as append + attention.  An empty
pool makes the append of the head that needs a page report device code 7 and
leave that head's context unchanged, while the other heads go on.
"""
from __future__ import annotations

import pytest
import torch

import oracle
from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _parity import assert_close, compare

pytestmark = pytest.mark.gpu

POOL_EMPTY = 7


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


def _bits(t):
    return t.view(torch.int16)


def _setup(N, spare, L0=(70, 200, 5, 131), cap=None):
    pol = []
    for _ in L0:
        pol += [("local", 4, 40), ("global", 0, 0), ("local", 0, 64), ("global", 0, 0)]
    hkv, g = 4, 2
    final = tuple(L + N for L in L0)
    wl = W.custom("spare", 91, len(L0), hkv * g, hkv, 128, "bf16", 64, final, pol)
    k, v = W.dense_kv(W.Problem(wl, final, tuple(L - 1 for L in final)), device="cuda")
    full = W.Problem(wl, final, tuple(L - 1 for L in L0))
    qall, qoff = W.queries(full, device="cuda"), full.q_offsets
    start = W.Problem(wl, L0, tuple(L - 1 for L in L0))
    layer = layer_for(start, flags=S.SP_FLAG_RING, append_capacity=cap or N, spare_pages=spare)
    layer.build(k, v)
    return wl, L0, pol, k, v, qall, qoff, layer, start


def _needed(L0, N, globals_per_seq=2):
    """Pages the GLOBAL heads need beyond their first ceil(L / 64) pages to hold L + N tokens."""
    return sum(globals_per_seq * (-(-(L + N) // 64) - -(-L // 64)) for L in L0)


def test_global_heads_grow_from_the_shared_pool():
    N, cap = 150, 1000  # records for 1000 more tokens per head, pages for the 150 steps taken
    need = _needed((70, 200, 5, 131), N)
    wl, L0, pol, k, v, qall, qoff, layer, start = _setup(N, need, cap=cap)
    reserved = layer_for(start, flags=S.SP_FLAG_RING, append_capacity=cap).sizes.num_pages
    assert layer.sizes.num_pages < reserved - 2 * need
    B = len(L0)
    for i in range(N):
        pos = [L + i for L in L0]
        kn = torch.stack([k[b, :, p] for b, p in enumerate(pos)]).contiguous()
        vn = torch.stack([v[b, :, p] for b, p in enumerate(pos)]).contiguous()
        q = torch.stack([qall[qoff[b] + 1 + i] for b in range(B)]).contiguous()
        layer.append(kn, vn)
        out, lse = layer.attention(q)
        if i in (0, 63, 64, 100, N - 1):
            torch.cuda.synchronize()
            prob = W.Problem(wl, tuple(p + 1 for p in pos), tuple(pos))
            assert_close(compare(prob, q, k, v, out, lse), "bf16")
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    final = tuple(L + N for L in L0)
    ko, vo = torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
    layer.gather(ko, vo)
    torch.cuda.synchronize()
    kb, vb, kob, vob = _bits(k.cpu()), _bits(v.cpu()), _bits(ko.cpu()), _bits(vo.cpu())
    for b, L in enumerate(final):
        for kv in range(4):
            kind, s, w = pol[b * 4 + kv]
            m = torch.from_numpy(oracle.stored_mask(kind, s, w, L, L - 1))
            assert torch.equal(kob[b, kv, :L][m], kb[b, kv, :L][m]), (b, kv)
            assert torch.equal(vob[b, kv, :L][m], vb[b, kv, :L][m]), (b, kv)
    # the pool is used up exactly, and the table can be restored (pool refilled)
    S.segpaged_table_write(layer.plan, layer.table.data_ptr(), layer.table.numel(),
                           torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()


def test_fused_step_takes_the_same_pages():
    N = 120
    need = _needed((70, 200, 5, 131), N)
    wl, L0, pol, k, v, qall, qoff, a, start = _setup(N, need)
    b_layer = layer_for(start, flags=S.SP_FLAG_RING, append_capacity=N, spare_pages=need)
    b_layer.build(k, v)
    B = len(L0)
    for i in range(N):
        pos = [L + i for L in L0]
        kn = torch.stack([k[b, :, p] for b, p in enumerate(pos)]).contiguous()
        vn = torch.stack([v[b, :, p] for b, p in enumerate(pos)]).contiguous()
        q = torch.stack([qall[qoff[b] + 1 + i] for b in range(B)]).contiguous()
        oa, la = a.decode_step(kn, vn, q)
        b_layer.append(kn, vn)
        ob, lb = b_layer.attention(q)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob) and torch.equal(la, lb), i
    assert a.device_status() == 0 and b_layer.device_status() == 0
    # pages are taken in a launch-order-dependent order: compare the caches through gather
    ka, va = torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
    kb2, vb2 = torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
    a.gather(ka, va)
    b_layer.gather(kb2, vb2)
    torch.cuda.synchronize()
    assert torch.equal(_bits(ka), _bits(kb2)) and torch.equal(_bits(va), _bits(vb2))


def test_empty_pool_skips_the_append_and_reports():
    """Only sequence 0 outgrows its pages: its two GLOBAL heads (120 tokens, two pages) need a third
    page at position 128; with a pool of one page one of them gets it, the other reports code 7 and
    keeps its context, and every other head goes on."""
    N = 20
    wl, L0, pol, k, v, qall, qoff, layer, start = _setup(N, 1, L0=(120, 10, 5, 3))
    B = len(L0)
    for i in range(N):
        pos = [L + i for L in L0]
        kn = torch.stack([k[b, :, p] for b, p in enumerate(pos)]).contiguous()
        vn = torch.stack([v[b, :, p] for b, p in enumerate(pos)]).contiguous()
        layer.append(kn, vn)
    torch.cuda.synchronize()
    assert layer.device_status() == POOL_EMPTY
    # the last decode: every head but the starved one holds all its tokens
    q = torch.stack([qall[qoff[b] + N] for b in range(B)]).contiguous()
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    pos = [L + N - 1 for L in L0]
    prob = W.Problem(wl, tuple(p + 1 for p in pos), tuple(pos))
    heads_ok = [h for h in range(8) if h // 2 not in (1, 3)]  # q-heads of sequence 0's local kv-heads
    assert_close(compare(prob, q, k, v, out, lse, heads=heads_ok, seqs=(0,)), "bf16")
    assert_close(compare(prob, q, k, v, out, lse, seqs=(1, 2, 3)), "bf16")
