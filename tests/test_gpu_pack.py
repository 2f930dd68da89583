"""build_segpaged_cache / segpaged_gather: bit-exact against the oracle's stored set."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_build_b200 import segpaged as S
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import layer_for
from _retrieval import oracle_head

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    S.load()


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def check_pack(prob, flags=0, **kw):
    """Pack, gather into a sentinel-filled dense buffer, and compare bit for bit."""
    wl = prob.wl
    k, v = W.dense_kv(prob)
    kd, vd = k.cuda(), v.cuda()
    layer = layer_for(prob, flags=flags, **kw)
    layer.build(kd, vd)
    ko = torch.full_like(kd, float("nan"))
    vo = torch.full_like(vd, float("nan"))
    layer.gather(ko, vo)
    torch.cuda.synchronize()
    kb, vb, kob, vob = _bits(k), _bits(v), _bits(ko.cpu()), _bits(vo.cpu())
    sentinel = _bits(torch.full((1,), float("nan"), dtype=k.dtype))[0]
    dense_masked = bool(flags & S.SP_FLAG_DENSE_MASKED)
    stored_total = 0
    for b in range(wl.batch):
        L, q0 = prob.ctx_lens[b], prob.q_starts[b]
        for kv in range(wl.num_kv_heads):
            kind, s, w, extra = oracle_head(prob, b, kv)
            m = oracle.stored_mask("global" if dense_masked else kind, s, w, L, q0, **extra)
            mt = torch.from_numpy(m)
            stored_total += int(m.sum())
            assert torch.equal(kob[b, kv, :L][mt], kb[b, kv, :L][mt]), (b, kv)
            assert torch.equal(vob[b, kv, :L][mt], vb[b, kv, :L][mt]), (b, kv)
            assert bool((kob[b, kv, :L][~mt] == sentinel).all()), (b, kv)
            assert bool((vob[b, kv, :L][~mt] == sentinel).all()), (b, kv)
    assert stored_total == layer.sizes.stored_token_heads
    return layer


def check_pack_full_size(prob):
    """check_pack at full size: inputs generated on the GPU, every comparison made there.

    The oracle's stored mask depends only on (kind, sink, window, L, q0): it is computed
    once per distinct key and reused for every (sequence, kv-head) that has it.
    """
    wl = prob.wl
    k, v = W.dense_kv(prob, device="cuda")
    layer = layer_for(prob)
    layer.build(k, v)
    ko = torch.full_like(k, float("nan"))
    vo = torch.full_like(v, float("nan"))
    layer.gather(ko, vo)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    kb, vb, kob, vob = _bits(k), _bits(v), _bits(ko), _bits(vo)
    sentinel = int(_bits(torch.full((1,), float("nan"), dtype=k.dtype))[0])
    masks, stored_total = {}, 0
    for b in range(wl.batch):
        L, q0 = prob.ctx_lens[b], prob.q_starts[b]
        for kv in range(wl.num_kv_heads):
            kind, s, w, extra = oracle_head(prob, b, kv)
            key = (kind, s, w, L, q0) if not extra else (b, kv)
            if key not in masks:
                masks[key] = torch.from_numpy(oracle.stored_mask(kind, s, w, L, q0, **extra)).cuda()
            mt = masks[key]
            stored_total += int(mt.sum())
            assert torch.equal(kob[b, kv, :L][mt], kb[b, kv, :L][mt]), (b, kv)
            assert torch.equal(vob[b, kv, :L][mt], vb[b, kv, :L][mt]), (b, kv)
            assert bool((kob[b, kv, :L][~mt] == sentinel).all()), (b, kv)
            assert bool((vob[b, kv, :L][~mt] == sentinel).all()), (b, kv)
    assert stored_total == layer.sizes.stored_token_heads
    return stored_total


# Stored token-heads in closed form (sink + window per local head, L per global head; a chunk of C
# queries adds C - 1 to each local head): Llama-70B-shaped 32K layer and MHA 128K layer.
FULL_SIZE_STORED = {("llama", "decode"): 721_120, ("llama", "prefill"): 950_440,
                    ("mha", "decode"): 4_223_872, ("mha", "prefill"): 5_141_152}


@pytest.mark.parametrize("name,mode", [("llama", "decode"), ("llama", "prefill"), ("mha", "decode"),
                                       ("mha", "prefill"), ("ragged", "decode")])
def test_pack_gather_bit_exact_at_full_size(name, mode):
    """Every stored row of the bench's 32K layer, the MHA 128K layer and the ragged batch, bit for bit."""
    wl = W.ALL[name]()
    prob = wl.decode_problem() if mode == "decode" else wl.prefill_problem()
    n = check_pack_full_size(prob)
    if (name, mode) in FULL_SIZE_STORED:
        assert n == FULL_SIZE_STORED[(name, mode)]
    else:  # ragged: per sequence 2 global heads of L tokens, 6 local heads of min(L, 4 + 512)
        assert n == sum(2 * L + 6 * min(L, 4 + 512) for L in prob.ctx_lens)


@pytest.mark.parametrize("name", ["tiny", "mistral"])
@pytest.mark.parametrize("mode", ["decode", "prefill"])
def test_pack_gather_bit_exact(name, mode):
    wl = W.ALL[name]()
    check_pack(wl.decode_problem() if mode == "decode" else wl.prefill_problem())


def test_pack_dense_masked_keeps_everything():
    check_pack(W.mistral().decode_problem(), flags=S.SP_FLAG_DENSE_MASKED)


def test_pack_with_permuted_pages_and_offset_pool():
    prob = W.tiny().decode_problem()
    n = layer_for(prob).sizes.num_pages
    perm = list(np.random.default_rng(1).permutation(n) * 2)  # sparse ids in a larger pool
    check_pack(prob, first_page=3, page_ids=perm)


@pytest.mark.parametrize("dtype,page,d", [("f32", 16, 64), ("f32", 64, 128), ("bf16", 64, 64), ("bf16", 64, 128)])
def test_pack_ragged_edge_policies(dtype, page, d):
    """Ragged lengths, partial pages, sink >= L, sink 0, window 1, windows wider than the context."""
    lens = (1, 5, 63, 64, 65, 200, 130)
    pol = []
    for b, L in enumerate(lens):
        pol += [("global", 0, 0), ("local", 4, 1), ("local", 0, 7), ("local", 70, 3), ("dense", 0, 0),
                ("local", 3, 1000)]
    wl = W.custom("edge", 11, len(lens), 6, 6, d, dtype, page, lens, pol, chunk=37)
    check_pack(wl.decode_problem())
    check_pack(wl.prefill_problem())


def test_pack_varlen_layout_matches_padded():
    wl = W.custom("var", 12, 3, 4, 2, 64, "bf16", 64, (100, 257, 64),
                  [("global", 0, 0), ("local", 4, 16)] * 3)
    prob = wl.decode_problem()
    k, v = W.dense_kv(prob)
    # varlen [sum L, Hkv, d]
    kvar = torch.cat([k[b, :, :L].transpose(0, 1) for b, L in enumerate(prob.ctx_lens)]).contiguous().cuda()
    vvar = torch.cat([v[b, :, :L].transpose(0, 1) for b, L in enumerate(prob.ctx_lens)]).contiguous().cuda()
    a = layer_for(prob)
    a.build(k.cuda(), v.cuda())
    bl = layer_for(prob)
    bl.build(kvar, vvar, varlen=True)
    torch.cuda.synchronize()
    assert torch.equal(a.k_pool, bl.k_pool) and torch.equal(a.v_pool, bl.v_pool)
    ko, vo = torch.zeros_like(kvar), torch.zeros_like(vvar)
    bl.gather(ko, vo, varlen=True)
    torch.cuda.synchronize()
    for b, L in enumerate(prob.ctx_lens):
        off = sum(prob.ctx_lens[:b])
        for kv in range(2):
            kind, s, w = wl.policy[b * 2 + kv]
            m = torch.from_numpy(oracle.stored_mask(kind, s, w, L, L - 1)).cuda()
            assert torch.equal(ko[off:off + L, kv][m], kvar[off:off + L, kv][m])
            assert torch.equal(vo[off:off + L, kv][m], vvar[off:off + L, kv][m])


def test_two_layers_share_one_pool_through_first_page():
    """Layers of a model keep their pages in one pool: layer 1 starts at layer 0's pool_pages."""
    l0 = W.llama(layer=0, batch=1)
    l1 = W.llama(layer=1, batch=1)
    p0, p1 = l0.decode_problem(), l1.decode_problem()
    a = layer_for(p0)
    n0 = a.sizes.pool_pages
    b = layer_for(p1, first_page=n0)
    pool_bytes = b.sizes.pool_pages * b.sizes.page_bytes
    kpool = torch.empty(pool_bytes, dtype=torch.uint8, device="cuda")
    vpool = torch.empty(pool_bytes, dtype=torch.uint8, device="cuda")
    a = layer_for(p0, pools=(kpool, vpool))
    b = layer_for(p1, first_page=n0, pools=(kpool, vpool))
    from _parity import assert_close, compare
    inputs = []
    for lay, prob in ((a, p0), (b, p1)):
        k, v = W.dense_kv(prob, device="cuda")
        lay.build(k, v)
        inputs.append((k, v, W.queries(prob, device="cuda")))
    for lay, prob, (k, v, q) in ((a, p0, inputs[0]), (b, p1, inputs[1])):
        out, lse = lay.attention(q)
        torch.cuda.synchronize()
        assert_close(compare(prob, q, k, v, out, lse), "bf16")


@pytest.mark.parametrize("kv_dtype", [None, "e4m3"])
def test_pack_several_layers_in_one_launch(kv_dtype):
    """build_segpaged_cache_layers: one launch for three layers sharing the pools gives the
    same pool bytes as three build_segpaged_cache calls, and every layer gathers back bit-exact."""
    from head_aware_paged_build_b200.runtime import build_layers
    probs = [W.llama(layer=i, batch=1).decode_problem() for i in range(3)]
    kw = lambda i: dict(kv_dtype="e4m3", k_scale=0.01 * (i + 1), v_scale=0.02 * (i + 1)) if kv_dtype else {}
    first, firsts = 0, []
    for i, prob in enumerate(probs):
        firsts.append(first)
        first += layer_for(prob, first_page=first, **kw(i)).sizes.pool_pages - first
    probe = layer_for(probs[0], **kw(0))
    nbytes = first * probe.sizes.page_bytes
    dense = [W.dense_kv(prob, device="cuda") for prob in probs]
    pools = []
    for one_launch in (True, False):
        kpool = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        vpool = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        layers = [layer_for(prob, first_page=f, pools=(kpool, vpool), **kw(i))
                  for i, (prob, f) in enumerate(zip(probs, firsts))]
        if one_launch:
            build_layers(layers, [k for k, _ in dense], [v for _, v in dense])
        else:
            for lay, (k, v) in zip(layers, dense):
                lay.build(k, v)
        torch.cuda.synchronize()
        pools.append((kpool, vpool, layers))
    assert torch.equal(pools[0][0], pools[1][0]) and torch.equal(pools[0][1], pools[1][1])
    if kv_dtype is None:
        for lay, prob, (k, v) in zip(pools[0][2], probs, dense):
            ko, vo = torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
            lay.gather(ko, vo)
            torch.cuda.synchronize()
            for kv in range(prob.wl.num_kv_heads):
                kind, s, w = prob.wl.policy[kv]
                L = prob.ctx_lens[0]
                m = torch.from_numpy(oracle.stored_mask(kind, s, w, L, L - 1)).cuda()
                assert torch.equal(_bits(ko[0, kv, :L][m]), _bits(k[0, kv, :L][m])), kv
                assert torch.equal(_bits(vo[0, kv, :L][m]), _bits(v[0, kv, :L][m])), kv
