"""FP8 E4M3 KV pages: codes bit-exact against the oracle's encoder, attention against the oracle.

The pages store E4M3(fp32(x) * (1 / scale)) per element with one scale for K
and one for V; the attention must equal the oracle's fp64 attention over the
decoded values code * scale (within the bf16 tolerances), and the codes must
equal the oracle's nearest-even, saturating encoder bit for bit.
"""
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

NAN_CODE = 0x7F  # never produced by the saturating encoder: marks untouched bytes


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


def amax_scale(x: torch.Tensor) -> float:
    """Per-tensor scale that maps the largest magnitude to 448 (the caller's choice, not the method's)."""
    return float(np.float32(float(x.float().abs().max()) / 448.0))


def oracle_codes(prob, dense: torch.Tensor, scale: float, dense_masked: bool = False):
    """Oracle codes and decoded values at every stored position (others: NAN_CODE and 0)."""
    wl = prob.wl
    inv = np.float32(1.0) / np.float32(scale)
    x = dense.float().cpu().numpy()
    codes = np.full(x.shape, NAN_CODE, np.uint8)
    vals = np.zeros(x.shape, np.float64)
    masks = {}
    for b in range(wl.batch):
        L, q0 = prob.ctx_lens[b], prob.q_starts[b]
        for kv in range(wl.num_kv_heads):
            kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
            m = oracle.stored_mask("global" if dense_masked else kind, s, w, L, q0)
            idx = np.nonzero(m)[0]
            c = oracle.e4m3_encode(x[b, kv, idx], inv)
            codes[b, kv, idx] = c
            vals[b, kv, idx] = oracle.e4m3_decode(c, scale)
            masks[b, kv] = m
    return codes, vals, masks


def fp8_layer(prob, k, v, ks, vs, **kw):
    layer = layer_for(prob, kv_dtype="e4m3", k_scale=ks, v_scale=vs, **kw)
    layer.build(k, v)
    return layer


def check_codes(layer, prob, k, v, ks, vs, dense_masked=False):
    ko = torch.full(k.shape, NAN_CODE, dtype=torch.uint8, device="cuda")
    vo = torch.full(v.shape, NAN_CODE, dtype=torch.uint8, device="cuda")
    layer.gather(ko, vo)
    torch.cuda.synchronize()
    kc, kvals, masks = oracle_codes(prob, k, ks, dense_masked)
    vc, vvals, _ = oracle_codes(prob, v, vs, dense_masked)
    assert np.array_equal(ko.cpu().numpy(), kc)
    assert np.array_equal(vo.cpu().numpy(), vc)
    assert sum(int(m.sum()) for m in masks.values()) == layer.sizes.stored_token_heads
    return kvals, vvals


def edge_workload(d):
    lens = (1, 5, 63, 64, 65, 200, 130)
    pol = []
    for _ in lens:
        pol += [("global", 0, 0), ("local", 4, 1), ("local", 0, 7), ("local", 70, 3), ("dense", 0, 0),
                ("local", 3, 1000)]
    return W.custom("fp8edge", 71, len(lens), 12, 6, d, "bf16", 64, lens, pol)


@pytest.mark.parametrize("case", ["edge64", "edge128", "mistral"])
def test_fp8_pack_and_decode_match_oracle(case):
    wl = {"edge64": lambda: edge_workload(64), "edge128": lambda: edge_workload(128)}.get(case, W.ALL.get(case))()
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    ks, vs = amax_scale(k), amax_scale(v)
    layer = fp8_layer(prob, k, v, ks, vs)
    kvals, vvals = check_codes(layer, prob, k, v, ks, vs)
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert_close(compare(prob, q, torch.from_numpy(kvals), torch.from_numpy(vvals), out, lse), "bf16")


def test_fp8_saturation_and_dense_masked():
    """A scale far below amax / 448: many codes saturate at +-448 on both sides; dense + mask keeps everything."""
    wl = W.mistral()
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    ks, vs = amax_scale(k) / 8, amax_scale(v) / 4
    layer = fp8_layer(prob, k, v, ks, vs, flags=S.SP_FLAG_DENSE_MASKED)
    kvals, vvals = check_codes(layer, prob, k, v, ks, vs, dense_masked=True)
    assert np.mean(np.abs(kvals) >= 448 * ks * (1 - 1e-9)) > 1e-3  # saturation really happens
    out, lse = layer.attention(q)
    torch.cuda.synchronize()
    assert_close(compare(prob, q, torch.from_numpy(kvals), torch.from_numpy(vvals), out, lse), "bf16")


def test_fp8_split_heads_merge_and_single_cta_agree():
    """Many CTAs per head (in-kernel merge) vs one item per head: both match the oracle."""
    wl = W.mistral()
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob, device="cuda")
    q = W.queries(prob, device="cuda")
    ks, vs = amax_scale(k), amax_scale(v)
    _, kvals, _ = oracle_codes(prob, k, ks)
    _, vvals, _ = oracle_codes(prob, v, vs)
    for target in (1, 2000):
        layer = fp8_layer(prob, k, v, ks, vs, target_ctas=target)
        out, lse = layer.attention(q)
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        assert_close(compare(prob, q, torch.from_numpy(kvals), torch.from_numpy(vvals), out, lse), "bf16")


@pytest.mark.parametrize("d,g", [(128, 4), (64, 1)])
def test_fp8_ring_appends_match_oracle(d, g):
    """Ring plan on E4M3 pages: every appended row is quantised like the pack; rings wrap several times."""
    L0 = (70, 200, 5, 131)
    N = 140
    pol = []
    for _ in L0:
        pol += [("local", 4, 40), ("global", 0, 0), ("local", 0, 64), ("local", 300, 10)]
    hkv = 4
    final = tuple(L + N for L in L0)
    wl = W.custom("ring8", 73, len(L0), hkv * g, hkv, d, "bf16", 64, final, pol)
    full = W.Problem(wl, final, tuple(L - 1 for L in final))
    k, v = W.dense_kv(full, device="cuda")
    ks, vs = amax_scale(k), amax_scale(v)
    qprob = W.Problem(wl, final, tuple(L - 1 for L in L0))
    qall, qoff = W.queries(qprob, device="cuda"), qprob.q_offsets
    layer = layer_for(W.Problem(wl, L0, tuple(L - 1 for L in L0)), flags=S.SP_FLAG_RING, append_capacity=N,
                      kv_dtype="e4m3", k_scale=ks, v_scale=vs)
    layer.build(k, v)
    # every position's decoded value (a position's code does not depend on which call stored it)
    all_pos = W.Problem(wl, final, tuple(0 for _ in final))
    kc_all, kvals, _ = oracle_codes(all_pos, k, ks, dense_masked=True)
    vc_all, vvals, _ = oracle_codes(all_pos, v, vs, dense_masked=True)
    out = torch.empty(len(L0), hkv * g, d, dtype=k.dtype, device="cuda")
    lse = torch.empty(len(L0), hkv * g, dtype=torch.float32, device="cuda")
    check = set(range(0, N, 13)) | {N - 1}
    for i in range(N):
        pos = [L + i for L in L0]
        layer.append(torch.stack([k[b, :, p] for b, p in enumerate(pos)]).contiguous(),
                     torch.stack([v[b, :, p] for b, p in enumerate(pos)]).contiguous())
        q = torch.stack([qall[qoff[b] + 1 + i] for b in range(len(L0))]).contiguous()
        layer.attention(q, out, lse)
        if i in check:
            torch.cuda.synchronize()
            prob = W.Problem(wl, tuple(p + 1 for p in pos), tuple(pos))
            assert_close(compare(prob, q, torch.from_numpy(kvals), torch.from_numpy(vvals), out, lse), "bf16")
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    ko = torch.full(k.shape, NAN_CODE, dtype=torch.uint8, device="cuda")
    vo = torch.full(v.shape, NAN_CODE, dtype=torch.uint8, device="cuda")
    layer.gather(ko, vo)
    torch.cuda.synchronize()
    ko, vo = ko.cpu().numpy(), vo.cpu().numpy()
    for b, L in enumerate(final):
        for kv in range(hkv):
            kind, s, w = pol[b * hkv + kv]
            m = oracle.stored_mask(kind, s, w, L, L - 1)
            assert np.array_equal(ko[b, kv, :L][m], kc_all[b, kv, :L][m]), (b, kv)
            assert np.array_equal(vo[b, kv, :L][m], vc_all[b, kv, :L][m]), (b, kv)
            assert (ko[b, kv, :L][~m] == NAN_CODE).all() and (vo[b, kv, :L][~m] == NAN_CODE).all(), (b, kv)
