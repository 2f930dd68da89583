"""Host-side pieces of bench.py that need no GPU: the sampled decode parity bookkeeping."""
from __future__ import annotations

import sys
from pathlib import Path

import numpy as np
import torch

import oracle
from head_aware_paged_build_b200 import workloads as W

sys.path.insert(0, str(Path(__file__).resolve().parent.parent))
import bench  # noqa: E402


def _oracle_decode(wl, dec, k, v, q):
    out = torch.zeros(q.shape, dtype=torch.float64)
    lse = torch.zeros(q.shape[:2], dtype=torch.float64)
    for b in range(wl.batch):
        L = dec.ctx_lens[b]
        for kv in range(wl.num_kv_heads):
            kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
            hs = slice(kv * wl.group, (kv + 1) * wl.group)
            o, l = oracle.attention_rows(q[b, hs].double().numpy(), [L - 1] * wl.group, k[b, kv, :L].double().numpy(),
                                         v[b, kv, :L].double().numpy(), kind, s, w)
            out[b, hs], lse[b, hs] = torch.from_numpy(o), torch.from_numpy(l)
    return out, lse


def test_sampled_parity_matches_and_catches_a_wrong_head():
    wl = W.tiny()
    dec = wl.decode_problem()
    k, v = W.dense_kv(dec)
    q = W.queries(dec)
    out, lse = _oracle_decode(wl, dec, k, v, q)
    _, vis, groups, par = bench.oracle_decode_sample(wl, dec, k, v, q, 1e9, gpu=(out, lse))
    assert groups == wl.batch * wl.num_kv_heads and par["heads"] == wl.num_q_heads
    assert par["min_cos"] >= 1 - 1e-12 and par["max_abs"] == 0.0 and par["max_lse_abs"] == 0.0
    assert vis == sum(int(oracle.stored_mask(kd, s, w, dec.ctx_lens[0], dec.ctx_lens[0] - 1).sum())
                      for kd, s, w in wl.policy) * 2 * wl.head_dim * 2
    bad = out.clone()
    bad[0, wl.num_q_heads - 1] = torch.from_numpy(np.roll(bad[0, wl.num_q_heads - 1].numpy(), 1))
    _, _, _, par = bench.oracle_decode_sample(wl, dec, k, v, q, 1e9, gpu=(bad, lse))
    assert par["min_cos"] < 0.99 and par["max_abs"] > 0
