"""Host-side pieces of bench.py that need no GPU: sampled decode parity, clocks record, traffic record, rates."""
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


def test_prefill_sample_rate_ledger_parity_and_cores():
    """The prefill CPU baseline: full run over the tiny layer's chunk counts every visible pair
    (the closed form 21,238,784 FLOPs), matches an oracle-made output exactly and reports the
    host's affinity core count; a planted wrong row is caught."""
    wl = W.tiny()
    pre = wl.prefill_problem()
    k, v = W.dense_kv(pre)
    q = W.queries(pre)
    out = torch.zeros(q.shape, dtype=torch.float64)
    lse = torch.zeros(q.shape[:2], dtype=torch.float64)
    L, q0 = pre.ctx_lens[0], pre.q_starts[0]
    for h in range(wl.num_q_heads):
        kind, s, w = wl.policy[h // wl.group]
        o, l = oracle.attention_rows(q[:, h].double().numpy(), np.arange(q0, L), k[0, h // wl.group, :L].double().numpy(),
                                     v[0, h // wl.group, :L].double().numpy(), kind, s, w)
        out[:, h], lse[:, h] = torch.from_numpy(o), torch.from_numpy(l)
    rec = bench.oracle_prefill_sample(wl, pre, k, v, q, 1e9, full=True, gpu=(out, lse))
    assert rec["extrapolated"] is False and rec["parity"]["rows"] == pre.total_queries * wl.num_q_heads
    assert rec["parity"]["max_abs"] == 0.0 and rec["parity"]["max_lse_abs"] == 0.0
    assert bench.pre_visible_pairs(wl, pre) * 4 * wl.head_dim == 21_238_784
    assert rec["cores"] == len(__import__("os").sched_getaffinity(0)) and rec["value"] > 0
    bad = out.clone()
    bad[5, 1] = -bad[5, 1]
    rec = bench.oracle_prefill_sample(wl, pre, k, v, q, 1e9, full=True, gpu=(bad, lse))
    assert rec["parity"]["min_cos"] < 0.999
    samp = bench.oracle_prefill_sample(wl, pre, k, v, q, 1e9, rows_per_head=8)
    assert samp["extrapolated"] is True and "8 seeded random rows" in samp["sample"]


def test_clock_sampler_takes_median_max_and_active_reasons():
    """The clocks record of the bench line, from nvidia-smi CSV rows (no GPU: a fake process)."""
    class Fake:
        def terminate(self):
            pass

        def communicate(self, timeout=None):
            rows = ["1800, 1965, 900.1, 0x4, Not Active, Not Active, Not Active, Active",
                    "1770, 1965, 950.3, 0x4, Not Active, Not Active, Not Active, Active",
                    "1500, 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active",
                    "[N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
                    "garbage"]
            return "\n".join(rows), ""

    cs = object.__new__(bench.ClockSampler)
    cs.proc = Fake()
    rec = cs.stop()
    assert rec == {"sm_mhz": 1770.0, "sm_max_mhz": 1965.0, "samples": 3, "reasons": ["sw_power_cap"]}
    cs.proc = None
    assert cs.stop() is None


def test_kernel_traffic_only_while_the_source_is_unchanged(tmp_path, monkeypatch):
    """DRAM bytes come from profiles/traffic.json only for the captured workload and kernel source."""
    import hashlib
    import json
    src = tmp_path / "kernel.cu"
    src.write_text("// a kernel\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k": {"bytes_per_launch": 123, "source_sha16": sha, "workload_key": "llama_l0"}}))
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    assert bench.kernel_traffic("k", src, "llama_l0") == 123
    assert bench.kernel_traffic("k", src, "llama_l0_other") is None
    assert bench.kernel_traffic("no_such_kernel", src, "llama_l0") is None
    src.write_text("// a kernel, changed\n")
    assert bench.kernel_traffic("k", src, "llama_l0") is None
    # the committed record names the bench's kernels and workload
    rec = json.loads((Path(__file__).resolve().parent.parent / "profiles" / "traffic.json").read_text())
    assert {"prefill_tc_kernel", "decode_mma_kernel"} <= set(rec)


def test_weak_rate_and_config():
    assert bench.weak_rate(1e9, 4, 2.0) == 4 * 1e9 / 2e-3
    cfg = bench.config_of(W.llama(), 1)
    assert cfg["workload"] == "Llama-70B-shaped layer, 32K context"
    assert cfg["heads"] == {"global": 8, "local": 56} and cfg["local_sink_window"] == [4, 8192]
    assert cfg["parallelism"] == "single GPU" and bench.config_of(W.llama(), 8)["parallelism"] == "replicas x8"
