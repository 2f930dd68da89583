"""RETRIEVAL heads on the GPU: packing bit for bit, decode and prefill against the fp64 oracle.

The planner chooses each retrieval head's kept blocks from the importance
inputs; the oracle makes its own choice from the same inputs and computes
dense attention with the explicit retrieval mask (sink, window, kept blocks).
"""
from __future__ import annotations

import pytest
import torch

from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _parity import assert_close, compare, sample_rows
from test_gpu_pack import check_pack
from test_retrieval_plan import edge_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


def run(prob, flags=0, device_inputs=False, **kw):
    gen = "cuda" if device_inputs else "cpu"
    k, v = W.dense_kv(prob, device=gen)
    q = W.queries(prob, device=gen)
    layer = layer_for(prob, flags=flags, **kw)
    layer.build(k.cuda(), v.cuda())
    out, lse = layer.attention(q.cuda())
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return layer, (k, v, q), out, lse


@pytest.mark.parametrize("mode", ["decode", "prefill"])
@pytest.mark.parametrize("flags", [0, S.SP_FLAG_DENSE_MASKED])
def test_tiny_retrieval_f32_matches_oracle(mode, flags):
    wl = W.tiny_retrieval()
    prob = wl.decode_problem() if mode == "decode" else wl.prefill_problem()
    _, (k, v, q), out, lse = run(prob, flags)
    assert_close(compare(prob, q, k, v, out, lse), "f32")


@pytest.mark.parametrize("dtype,page,d", [("bf16", 64, 128), ("bf16", 64, 64), ("f32", 16, 64), ("f32", 64, 128)])
@pytest.mark.parametrize("mode", ["decode", "prefill"])
@pytest.mark.parametrize("flags", [0, S.SP_FLAG_DENSE_MASKED])
def test_retrieval_edge_policies_match_oracle(dtype, page, d, mode, flags):
    """Context 1 .. 700, sink 0 .. 70, window 1 .. 1000, top_p 0 .. 1, ragged chunk of 140 queries."""
    wl = edge_workload(dtype, page, d)
    prob = wl.decode_problem() if mode == "decode" else wl.prefill_problem()
    _, (k, v, q), out, lse = run(prob, flags)
    assert_close(compare(prob, q, k, v, out, lse), dtype)


@pytest.mark.parametrize("mode", ["decode", "prefill"])
def test_retrieval_pack_gather_bit_exact(mode):
    for wl in (W.tiny_retrieval(), edge_workload(), edge_workload("f32", 16, 64)):
        check_pack(wl.decode_problem() if mode == "decode" else wl.prefill_problem())


def test_retrieval_top_p_one_is_bitwise_global():
    """top_p = 1 keeps every block: the same pages as a GLOBAL head, every page seen causally."""
    lens = (3000, 1000)
    glob = W.custom("tp1", 63, 2, 8, 2, 128, "bf16", 64, lens, [("global", 0, 0), ("local", 4, 300)] * 2,
                    chunk=700)
    retr = W.custom("tp1", 63, 2, 8, 2, 128, "bf16", 64, lens,
                    [("retrieval", 4, 300, 1.0), ("local", 4, 300)] * 2, chunk=700)
    for mode in ("decode", "prefill"):
        pg = glob.decode_problem() if mode == "decode" else glob.prefill_problem()
        pr = retr.decode_problem() if mode == "decode" else retr.prefill_problem()
        _, _, og, lg = run(pg)
        _, (k, v, q), orr, lr = run(pr)
        assert torch.equal(og, orr) and torch.equal(lg, lr), mode
        assert_close(compare(pr, q, k, v, orr, lr), "bf16")


def test_retrieval_decode_e4m3_pages_match_oracle_on_decoded_values():
    import numpy as np

    import oracle
    wl = W.llama_retrieval(batch=2)
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    ks, vs = float(k.float().abs().max()) / 448, float(v.float().abs().max()) / 448
    layer = layer_for(prob, kv_dtype="e4m3", k_scale=ks, v_scale=vs)
    layer.build(k, v)
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    # attention is defined on the decoded values code * scale
    kvals = oracle.e4m3_decode(oracle.e4m3_encode(k.float().cpu().numpy(), np.float32(1 / ks)), ks)
    vvals = oracle.e4m3_decode(oracle.e4m3_encode(v.float().cpu().numpy(), np.float32(1 / vs)), vs)
    assert_close(compare(prob, q, torch.from_numpy(kvals), torch.from_numpy(vvals), out, lse), "bf16")


@pytest.mark.parametrize("mode", ["decode", "prefill"])
def test_llama_retrieval_layer_matches_oracle(mode):
    """The 32K layer with two retrieval kv-heads per sequence (batch 2), every q-head; prefill rows at
    chunk edges, tile edges +-1 and seeded random rows."""
    wl = W.llama_retrieval(batch=2)
    prob = wl.decode_problem() if mode == "decode" else wl.prefill_problem()
    _, (k, v, q), out, lse = run(prob, device_inputs=True)
    rows = None if mode == "decode" else [sample_rows(c, stride=256, n_random=8, seed=b)
                                          for b, c in enumerate(prob.q_counts)]
    assert_close(compare(prob, q, k, v, out, lse, rows_per_seq=rows), "bf16")
