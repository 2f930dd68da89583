"""segpaged_block_mass: the attention mass per page-size block (a retrieval head's importance).

Each (sequence, kv-head) row is compared with the fp64 oracle's block mass of
the same keys and queries: every entry within 2e-4 relative + 1e-7 absolute
(fp32 scores of bf16 products, fp32 sums), rows summing to 1, zeros after a
row's blocks.  Shapes: the Llama-70B-shaped 32K layer at batch 8, head_dim 64
with 16 q-heads per kv-head, one q-head per kv-head, ragged lengths (1, one
block, one position past a block, a partial last block), contexts past 512
blocks (the normalisation then takes a row in several passes), keys read through
a [B, L, Hkv, d] layout; repeated calls are bitwise equal.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_build_b200 import workloads as W
from head_aware_paged_build_b200.runtime import block_mass

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _inputs(name, seed, B, hq, hkv, d, lens):
    wl = W.custom(name, seed, B, hq, hkv, d, "bf16", 64, lens, [("global", 0, 0)] * (B * hkv))
    prob = wl.decode_problem()  # one query per sequence, at its last position
    k, _ = W.dense_kv(prob, device="cuda", gen_device="cuda")
    q = W.queries(prob, device="cuda", gen_device="cuda")
    return wl, k, q


def _check(m, k, q, lens, hkv):
    mh, kh, qh = m.cpu().double().numpy(), k.cpu(), q.cpu()
    g = q.shape[1] // hkv
    for b, L in enumerate(lens):
        nb = -(-L // 64)
        for kv in range(hkv):
            ref = oracle.block_mass(qh[b, kv * g:(kv + 1) * g].double().numpy(), kh[b, kv, :L].double().numpy(), 64)
            got = mh[b, kv]
            assert np.all(np.abs(got[:nb] - ref) <= 2e-4 * ref + 1e-7), (b, kv, np.abs(got[:nb] - ref).max())
            assert abs(got[:nb].sum() - 1.0) < 1e-5 and not got[nb:].any(), (b, kv)


@pytest.mark.parametrize("name,B,hq,hkv,d,lens", [
    ("mass_llama", 8, 64, 8, 128, (32768,) * 8),
    ("mass_d64_g16", 2, 32, 2, 64, (4000, 1500)),
    ("mass_mha", 2, 4, 4, 128, (3000, 700)),
    ("mass_ragged", 5, 16, 4, 128, (1, 64, 65, 130, 1999)),
    ("mass_long", 2, 8, 2, 128, (40000, 70001)),  # rows of more than 512 blocks
])
def test_block_mass_matches_oracle(name, B, hq, hkv, d, lens):
    wl, k, q = _inputs(name, 11, B, hq, hkv, d, lens)
    m = block_mass(k, q, lens)
    torch.cuda.synchronize()
    _check(m, k, q, lens, hkv)
    assert torch.equal(m, block_mass(k, q, lens))  # fixed summation orders: bitwise repeatable


def test_block_mass_reads_any_key_layout():
    """Keys laid out [B, L, Hkv, d] (token-major), read through the strides, give the same masses bit for bit."""
    lens = (777, 1290)
    wl, k, q = _inputs("mass_layout", 12, 2, 8, 2, 128, lens)
    tok_major = k.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)  # same values, strides (L Hkv d, d, Hkv d)
    assert tok_major.stride(1) == 128 and tok_major.stride(2) == 2 * 128
    m = block_mass(tok_major, q, lens)
    assert torch.equal(m, block_mass(k, q, lens))
    _check(m, k, q, lens, 2)


def test_gpu_scores_choose_the_oracles_blocks():
    """Scoring on the GPU, top-p selection by the planner, attention on the GPU, against the oracle's
    own scoring and selection from the same keys and queries.

    For each sequence's retrieval head, top_p sits halfway between two steps of the oracle's
    cumulative block mass where the blocks on either side differ by more than 1 %, so the GPU's
    masses (within 2e-4 of the oracle's) pick the same blocks: the plan's stored positions must
    equal the oracle's, and the decode output must match the oracle's attention over them.
    """
    import numpy as np

    from head_aware_paged_build_b200.runtime import layer_for
    from test_retrieval_plan import _held

    lens, B, hq, hkv, d, g = (3000, 4500), 2, 8, 2, 128, 4
    pol = [("retrieval", 4, 256, 1.0), ("local", 4, 256)] * B
    wl0 = W.custom("score_select", 13, B, hq, hkv, d, "bf16", 64, lens, pol)
    k, v = W.dense_kv(wl0.decode_problem(), device="cuda", gen_device="cuda")
    q = W.queries(wl0.decode_problem(), device="cuda", gen_device="cuda")
    kh, vh, qh = k.cpu().double().numpy(), v.cpu().double().numpy(), q.cpu().double().numpy()
    sels = {}
    for b, L in enumerate(lens):
        om = oracle.block_mass(qh[b, :g], kh[b, 0, :L], 64)  # kv-head 0 is the retrieval head
        srt = np.sort(om)[::-1]
        cum = np.cumsum(srt) / srt.sum()
        gap = (srt[:-1] - srt[1:]) / srt[:-1]  # gap[i]: the (i+1)-th largest mass vs the (i+2)-th
        # keep c blocks: top_p halfway between the shares of the top c - 1 and the top c blocks,
        # with the c-th and (c+1)-th largest masses more than 1 % apart
        c = next(c for c in range(5, len(srt) - 1) if gap[c - 1] > 0.01 and cum[c - 1] < 0.9)
        top_p = float(np.float32((cum[c - 2] + cum[c - 1]) / 2))
        pol[b * hkv] = ("retrieval", 4, 256, top_p)
        sels[b] = oracle.retrieval_select(L, 64, 4, top_p, om.astype(np.float32))
        assert sels[b].sum() == c
    wl = W.custom("score_select", 13, B, hq, hkv, d, "bf16", 64, lens, pol)  # same draws, chosen top_p
    prob = wl.decode_problem()
    m = block_mass(k, q, lens)
    masses = [m[b, kv, :-(-L // 64)].tolist() if kv == 0 else None for b, L in enumerate(lens) for kv in range(hkv)]
    layer = layer_for(prob, block_mass=masses)
    layer.build(k, v)
    out, _ = layer.attention(q)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    out = out.float().cpu().double().numpy()
    for b, L in enumerate(lens):
        held = _held(layer.plan, b, 0, L)
        assert np.array_equal(held, oracle.stored_mask("retrieval", 4, 256, L, L - 1, sel=sels[b], block=64)), b
        for h in range(hq):
            kv = h // g
            kind, s, w = pol[b * hkv + kv][:3]
            extra = dict(sel=sels[b], block=64) if kind == "retrieval" else {}
            ref, _ = oracle.attention_rows(qh[b, h][None], np.array([L - 1]), kh[b, kv, :L], vh[b, kv, :L], kind, s, w,
                                           **extra)
            o = out[b, h][None]
            cos = float((o * ref).sum() / (np.linalg.norm(o) * np.linalg.norm(ref)))
            assert cos >= 0.99998 and float(np.abs(o - ref).max()) <= 2e-2, (b, h, cos)
