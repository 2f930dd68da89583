"""segpaged_attention_decode_noalloc: decode without a caller workspace.

Callers whose device memory is fully assigned before they start (a fixed
arena), or who must not call cudaMalloc in their hot loop because it can
synchronise the device, use this entry point; its scratch is an array built
into the library.  The tests check, through the C ABI, that two calls in a
row give bit for bit the output of segpaged_attention with a workspace (same
plan, same kernels: only the scratch base differs), for bf16 pages, E4M3
pages and an fp32 plan (whose split heads merge in a separate combine pass);
that the leftovers of a call on a larger plan do not leak into the next call;
that a device-side error reaches the caller's status word; and that plans
the built-in scratch cannot hold, prefill plans and a missing status word are
refused before any launch.  The file sits last in collection order.
"""
from __future__ import annotations

import pytest
import torch

from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _table import BAD_PAGE, corrupt, global_head

pytestmark = pytest.mark.gpu


def _setup(name: str, **kw):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    wl = W.ALL[name.split("-")[0]]()
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    if name.endswith("e4m3"):  # E4M3 pages, per-tensor scales amax / 448
        kw.update(kv_dtype="e4m3", k_scale=float(k.float().abs().max()) / 448,
                  v_scale=float(v.float().abs().max()) / 448)
    layer = layer_for(prob, **kw)
    layer.build(k, v)
    return wl, layer, q


def _noalloc(layer, q, d_status):
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device=q.device)
    S.segpaged_attention_decode_noalloc(layer.plan, layer.table.data_ptr(), layer.k_pool.data_ptr(),
                                        layer.v_pool.data_ptr(), q.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                        0.0, d_status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return out, lse


@pytest.mark.parametrize("name", ["mistral", "ragged", "mistral-e4m3", "tiny"])
def test_noalloc_decode_equals_workspace_decode_twice(name):
    wl, layer, q = _setup(name)
    ref_o, ref_l = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert layer.sizes.num_combine > 0  # some heads are split: the scratch holds partials
    d_status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out, lse = _noalloc(layer, q, d_status)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    assert int(d_status.item()) == 0


def test_noalloc_leftovers_of_a_larger_plan_do_not_leak():
    """A plan with many split heads fills the scratch with its partials; the next plan's result is unchanged."""
    _, small, qs = _setup("mistral")
    ref_o, ref_l = small.attention(qs)
    _, big, qb = _setup("ragged", target_ctas=1500)  # 3.75 MiB of scratch: 5x the small plan
    assert big.sizes.workspace_bytes > small.sizes.workspace_bytes
    d_status = torch.zeros(1, dtype=torch.int32, device="cuda")
    big_ref = big.attention(qb)
    for _ in range(2):
        out, lse = _noalloc(big, qb, d_status)
        torch.cuda.synchronize()
        assert torch.equal(out, big_ref[0]) and torch.equal(lse, big_ref[1])
        out, lse = _noalloc(small, qs, d_status)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    assert int(d_status.item()) == 0


def test_noalloc_reports_a_page_outside_the_pool_in_the_callers_status_word():
    wl, layer, q = _setup("mistral")
    ref_o, ref_l = layer.attention(q)
    torch.cuda.synchronize()
    kv = global_head(wl)
    corrupt(layer, 0, kv, 3)
    d_status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = _noalloc(layer, q, d_status)
    torch.cuda.synchronize()
    assert int(d_status.item()) == BAD_PAGE
    g = wl.group
    bad = torch.zeros(q.shape[0], q.shape[1], dtype=torch.bool)
    bad[0, kv * g:(kv + 1) * g] = True
    assert torch.equal(out.cpu()[~bad], ref_o.cpu()[~bad])
    # restored table, cleared word: the exact result again
    S.segpaged_table_write(layer.plan, layer.table.data_ptr(), layer.table.numel(),
                           torch.cuda.current_stream().cuda_stream)
    d_status.zero_()
    out, lse = _noalloc(layer, q, d_status)
    torch.cuda.synchronize()
    assert int(d_status.item()) == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_noalloc_refuses_before_any_launch():
    lib = S.load()
    fake = 16  # never dereferenced: every case is refused on the host
    big = layer_for(W.llama().decode_problem(), target_ctas=100000)  # one item per page: ~47 MB of partials
    assert big.sizes.workspace_bytes > 4 << 20
    st = lib.segpaged_attention_decode_noalloc(big.plan, big.table.data_ptr(), big.k_pool.data_ptr(),
                                               big.v_pool.data_ptr(), fake, fake, None, 0.0, fake, None)
    assert st == S.SP_ERR_WORKSPACE and "scratch" in S.last_error()
    pre = layer_for(W.tiny().prefill_problem())
    st = lib.segpaged_attention_decode_noalloc(pre.plan, pre.table.data_ptr(), pre.k_pool.data_ptr(),
                                               pre.v_pool.data_ptr(), fake, fake, None, 0.0, fake, None)
    assert st == S.SP_ERR_UNSUPPORTED
    dec = layer_for(W.tiny().decode_problem())
    st = lib.segpaged_attention_decode_noalloc(dec.plan, dec.table.data_ptr(), dec.k_pool.data_ptr(),
                                               dec.v_pool.data_ptr(), fake, fake, None, 0.0, None, None)
    assert st == S.SP_ERR_INVALID_ARG and "d_status" in S.last_error()
    st = lib.segpaged_attention_decode_noalloc(dec.plan, dec.table.data_ptr(), dec.k_pool.data_ptr(),
                                               dec.v_pool.data_ptr(), fake, fake, None, float("inf"), fake, None)
    assert st == S.SP_ERR_INVALID_ARG and "softmax_scale" in S.last_error()
