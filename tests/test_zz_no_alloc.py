"""segpaged_attention_decode_noalloc: decode without a caller workspace.

Callers whose device memory is fully assigned before they start (a fixed
arena), or who must not call cudaMalloc in their hot loop, use this entry
point; its scratch is an array built into the library.  The test checks,
through the C ABI, that two calls in a row give the same results as
segpaged_attention with a workspace (within the bf16 tolerance of the parity
tests), and that a plan needing more than the built-in scratch is refused
before any launch.  It sits in its own file so that pytest collects it last.
"""
from __future__ import annotations

import pytest
import torch

from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _parity import TOL

pytestmark = pytest.mark.gpu


def _close(a: torch.Tensor, b: torch.Tensor, tol_abs: float, cos_min: float) -> None:
    a, b = a.double().flatten(), b.double().flatten()
    assert float((a - b).abs().max()) <= tol_abs
    assert float(a @ b / (a.norm() * b.norm())) >= cos_min


@pytest.mark.parametrize("name", ["mistral", "ragged", "mistral-e4m3"])
def test_noalloc_decode_matches_workspace_decode_twice(name):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    wl = W.ALL[name.split("-")[0]]()
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    if name.endswith("e4m3"):  # E4M3 pages, per-tensor scales amax / 448
        layer = layer_for(prob, kv_dtype="e4m3", k_scale=float(k.float().abs().max()) / 448,
                          v_scale=float(v.float().abs().max()) / 448)
    else:
        layer = layer_for(prob)
    layer.build(k, v)
    ref_o, ref_l = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    tol = TOL[wl.dtype]
    stream = torch.cuda.current_stream().cuda_stream
    d_status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full(ref_l.shape, float("nan"), dtype=torch.float32, device="cuda")
        S.segpaged_attention_decode_noalloc(layer.plan, layer.table.data_ptr(), layer.k_pool.data_ptr(),
                                            layer.v_pool.data_ptr(), q.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                            0.0, d_status.data_ptr() if call else None, stream)
        torch.cuda.synchronize()
        _close(out, ref_o, tol["abs"], tol["cos"])
        assert float((lse - ref_l).abs().max()) <= tol["lse"]
    assert int(d_status.item()) == 0


def test_noalloc_refuses_plans_beyond_its_scratch_and_prefill_plans():
    wl = W.llama()
    big = layer_for(wl.decode_problem(), target_ctas=100000)  # one item per page: ~47 MB of partials
    assert big.sizes.workspace_bytes > 4 << 20
    lib = S.load()
    st = lib.segpaged_attention_decode_noalloc(big.plan, big.table.data_ptr(), big.k_pool.data_ptr(),
                                               big.v_pool.data_ptr(), 16, 16, None, 0.0, None, None)
    assert st == S.SP_ERR_WORKSPACE and "scratch" in S.last_error()
    pre = layer_for(W.tiny().prefill_problem())
    st = lib.segpaged_attention_decode_noalloc(pre.plan, pre.table.data_ptr(), pre.k_pool.data_ptr(),
                                               pre.v_pool.data_ptr(), 16, 16, None, 0.0, None, None)
    assert st == S.SP_ERR_UNSUPPORTED
