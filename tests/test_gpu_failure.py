"""Device-side failure detection without a GPU fault.

A page id in the device table that lies outside the plan's pool is caught by
the kernels' own bounds check: nothing is read or written at that page, the
device status word says 5, and the context stays usable.  In the prefill
kernel the producer stops at such a page, so the other roles' bounded waits
run out (about a second or two each): the kernel still ends, with the status
set.  No test here faults, traps or hangs a GPU.
"""
from __future__ import annotations

import pytest
import torch

from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _parity import assert_close, compare
from _table import BAD_PAGE, corrupt, global_head

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


@pytest.mark.parametrize("kv_dtype", [None, "e4m3"])
def test_decode_reports_a_page_outside_the_pool(kv_dtype):
    wl = W.mistral()
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    kw = dict(kv_dtype="e4m3", k_scale=0.02, v_scale=0.02) if kv_dtype else {}
    layer = layer_for(prob, **kw)
    layer.build(k, v)
    ref_o, ref_l = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    kv = global_head(wl)
    corrupt(layer, 0, kv, 3)
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == BAD_PAGE
    # every other head is untouched (bitwise); the corrupted head lost only that page
    g = wl.group
    bad = torch.zeros(q.shape[0], q.shape[1], dtype=torch.bool)
    bad[0, kv * g:(kv + 1) * g] = True
    assert torch.equal(out.cpu()[~bad], ref_o.cpu()[~bad])
    assert torch.equal(lse.cpu()[~bad], ref_l.cpu()[~bad])
    assert bool(torch.isfinite(out.float()).all())
    # the context stays usable: restore the table and the result comes back
    S.segpaged_clear_device_status(layer.workspace.data_ptr(), torch.cuda.current_stream().cuda_stream)
    S.segpaged_table_write(layer.plan, layer.table.data_ptr(), layer.table.numel(),
                           torch.cuda.current_stream().cuda_stream)
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_append_writes_nothing_at_a_page_outside_the_pool():
    wl = W.custom("bad_append", 81, 2, 4, 2, 128, "bf16", 64, (100, 70), [("global", 0, 0), ("local", 4, 16)] * 2)
    prob = W.Problem(wl, (90, 60), (89, 59))
    k, v = W.dense_kv(W.Problem(wl, (100, 70), (99, 69)), device="cuda")
    layer = layer_for(prob, flags=S.SP_FLAG_RING, append_capacity=8)
    layer.build(k, v)
    torch.cuda.synchronize()
    # sequence 0's global head appends position 90 into its page 1; point that page outside the pool
    corrupt(layer, 0, 0, 1)
    kpool, vpool = layer.k_pool.clone(), layer.v_pool.clone()
    layer.append(k[:, :, 90].contiguous(), v[:, :, 90].contiguous())  # one token per sequence (positions 90, 60)
    torch.cuda.synchronize()
    assert layer.device_status() == BAD_PAGE
    # the other heads did append: the pools changed, but never at the corrupted head's pages
    assert not (torch.equal(layer.k_pool, kpool) and torch.equal(layer.v_pool, vpool))
    pb = layer.sizes.page_bytes
    for pid in S.segpaged_plan_head_pages(layer.plan, 0, 0):
        assert torch.equal(layer.k_pool[pid * pb:(pid + 1) * pb], kpool[pid * pb:(pid + 1) * pb])
        assert torch.equal(layer.v_pool[pid * pb:(pid + 1) * pb], vpool[pid * pb:(pid + 1) * pb])


def test_prefill_ends_with_a_status_when_its_producer_stops():
    """The producer meets a page outside the pool and stops; the MMA and softmax waits run out and end the kernel."""
    wl = W.custom("bad_prefill", 82, 1, 4, 2, 128, "bf16", 64, (600,), [("global", 0, 0), ("local", 4, 64)])
    prob = wl.prefill_problem() if wl.prefill_chunk else W.Problem(wl, (600,), (0,))
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    layer = layer_for(prob)
    layer.build(k, v)
    ref_o, ref_l = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert_close(compare(prob, q, k, v, ref_o, ref_l), "bf16")
    corrupt(layer, 0, 0, 4)
    out = torch.full_like(ref_o, float("nan"))
    out, lse = layer.attention(q, out)
    torch.cuda.synchronize()  # returns: every wait in the kernel is bounded
    assert layer.device_status() == BAD_PAGE
    # the context is still usable afterwards
    S.segpaged_clear_device_status(layer.workspace.data_ptr(), torch.cuda.current_stream().cuda_stream)
    S.segpaged_table_write(layer.plan, layer.table.data_ptr(), layer.table.numel(),
                           torch.cuda.current_stream().cuda_stream)
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
