"""Helpers of the GPU parity tests: run the oracle on the exact inputs the GPU used."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from _retrieval import oracle_head

# Tolerances of the attention outputs against the fp64 oracle: per-head
# cosine >= 0.99998 ("SegPagedAttention runtime design", §4 verify_against_dense)
# and a max absolute error of 1e-5 for fp32 inputs, 2e-2 for bf16 inputs (fp32
# accumulation in both).  LSE: 1e-5 (fp32); 2e-3 (bf16): scores are exact
# products of bf16 values summed in fp32 (relative error ~d * 2^-24) and the
# softmax sums use the unrounded fp32 weights, so the bf16 LSE error is set by
# fp32 accumulation and the SFU exp2, far below 2e-3 at |s| < 60.
TOL = {"f32": dict(cos=0.99998, abs=1e-5, lse=1e-5), "bf16": dict(cos=0.99998, abs=2e-2, lse=2e-3)}


def oracle_rows(prob, q_host, k_host, v_host, b, h, rows=None):
    """Oracle output for (sequence b, q-head h) at varlen rows `rows` (indices within the sequence)."""
    wl = prob.wl
    kv = h // wl.group
    kind, s, w, extra = oracle_head(prob, b, kv)
    L, q0 = prob.ctx_lens[b], prob.q_starts[b]
    C = L - q0
    rows = np.arange(C) if rows is None else np.asarray(rows)
    off = prob.q_offsets[b]
    # inputs may live on the GPU (large layers are generated there): copy the slices
    q = q_host[torch.as_tensor(off + rows, device=q_host.device), h].cpu().double().numpy()
    k = k_host[b, kv, :L].cpu().double().numpy()
    v = v_host[b, kv, :L].cpu().double().numpy()
    return oracle.attention_rows(q, q0 + rows, k, v, kind, s, w, **extra)


def compare(prob, q_host, k_host, v_host, out, lse, rows_per_seq=None, heads=None, seqs=None):
    """Compare GPU out / lse (device or host tensors) with the oracle.

    The checked (sequence, q-head, rows) go to the oracle grouped by kv-head, several
    kv-heads per batched call (all host cores; at most ~2 GB of fp64 K/V at a time).
    Returns dict(min_cos, max_abs, max_lse, worst) over the checked (b, h).
    """
    wl = prob.wl
    out_h = out.float().cpu()
    lse_h = lse.float().cpu() if lse is not None else None
    heads = range(wl.num_q_heads) if heads is None else heads
    tasks = {}  # (b, kv) -> [(h, rows)]
    for b in (range(wl.batch) if seqs is None else seqs):
        rows = None if rows_per_seq is None else rows_per_seq[b]
        if rows is not None and len(rows) == 0:
            continue
        C = prob.ctx_lens[b] - prob.q_starts[b]
        ridx = np.arange(C) if rows is None else np.asarray(rows)
        for h in heads:
            tasks.setdefault((b, h // wl.group), []).append((h, ridx))
    min_cos, max_abs, max_lse, worst = 1.0, 0.0, 0.0, None
    keys = list(tasks)
    budget = 2e9
    i = 0
    while i < len(keys):
        chunk, used = [], 0
        while i < len(keys) and (not chunk or used + 16 * prob.ctx_lens[keys[i][0]] * wl.head_dim <= budget):
            chunk.append(keys[i])
            used += 16 * prob.ctx_lens[keys[i][0]] * wl.head_dim
            i += 1
        groups, meta = [], []
        masses = prob.block_masses() if wl.has_retrieval else None
        for b, kv in chunk:
            kind, s, w, extra = oracle_head(prob, b, kv, masses)
            ext = (extra["sel"], extra["block"]) if extra else ()
            L, q0 = prob.ctx_lens[b], prob.q_starts[b]
            off = prob.q_offsets[b]
            k = k_host[b, kv, :L].cpu().double().numpy()
            v = v_host[b, kv, :L].cpu().double().numpy()
            for h, ridx in tasks[(b, kv)]:
                # inputs may live on the GPU (large layers are generated there): copy the slices
                q = q_host[torch.as_tensor(off + ridx, device=q_host.device), h].cpu().double().numpy()
                groups.append((q, q0 + ridx, k, v, kind, s, w) + ext)
                meta.append((b, h, off + ridx))
        res = oracle.attention_batch(groups)
        for (b, h, idx), (o_ref, l_ref) in zip(meta, res):
            o = out_h[idx, h].double().numpy()
            a, r = o.ravel(), o_ref.ravel()
            cos = float(a @ r / (np.linalg.norm(a) * np.linalg.norm(r)))
            err = float(np.max(np.abs(o - o_ref)))
            if cos < min_cos:
                min_cos, worst = cos, (b, h)
            max_abs = max(max_abs, err)
            if lse_h is not None:
                max_lse = max(max_lse, float(np.max(np.abs(lse_h[idx, h].double().numpy() - l_ref))))
    return dict(min_cos=min_cos, max_abs=max_abs, max_lse=max_lse, worst=worst)


def assert_close(res, dtype):
    tol = TOL[dtype]
    assert res["min_cos"] >= tol["cos"], res
    assert res["max_abs"] <= tol["abs"], res
    assert res["max_lse"] <= tol["lse"], res


def sample_rows(C: int, stride: int = 128, n_random: int = 16, seed: int = 0) -> np.ndarray:
    """First / last rows, rows at multiples of `stride` and one either side (tile edges), seeded random rows."""
    rng = np.random.default_rng(seed)
    pick = {0, 1, C - 1, C - 2}
    for m in range(stride, C, stride):
        pick.update((m - 1, m, m + 1))
    pick.update(int(x) for x in rng.integers(0, C, n_random))
    return np.array(sorted(x for x in pick if 0 <= x < C))
