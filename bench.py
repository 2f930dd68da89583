"""Benchmark of the SegPaged hot path on synthetic layers (one JSON line).

One step = one pass of the whole path over one batch: build_segpaged_cache
for the decode layout, decode attention, build_segpaged_cache for the
prefill-chunk layout, prefill attention.  Inputs are resident in HBM; L2 is
flushed (256 MB written, then 512 MB read so no dirty line is written back
inside a timed kernel) before every timed kernel; each kernel is timed with
CUDA events on the stream it is launched on.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama|mistral|mha|ragged|llama_b1]
    python bench.py --impl reference ...   # the CPU oracle, timed on the host cores

Under torchrun each rank runs its own batch (a different seed) on its own GPU:
weak scaling with no collective on the data path; the timing is the max over
ranks.  `value` is the decode visible-KV throughput; prefill TFLOP/s, the
packing rate and the dense-plus-mask variant are reported beside it, with the
serving decode step through the public API with pinned host buffers (`e2e`),
E4M3 pages, and, on the Llama-shaped layers, a layer with retrieval heads
(decode, prefill and the scoring pass that gives them their importance).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "SegPaged decode visible-KV GB/s (% HBM peak); prefill visible TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def workload(name: str, rank: int):
    from head_aware_paged_build_b200 import workloads as W
    wl = W.ALL[name]()
    # weak scaling: every rank runs the same layer shape on its own batch
    return dataclasses.replace(wl, seed=wl.seed + 7919 * rank) if rank else wl


def config_of(wl, n_gpus: int) -> dict:
    kinds = {}
    for k, s, w in wl.policy:
        kinds[k] = kinds.get(k, 0) + 1
    loc = next(((s, w) for k, s, w in wl.policy if k == "local"), None)
    return {
        "workload": ("Llama-70B-shaped layer, 32K context" if wl.name.startswith("llama")
                     else {"mistral": "Mistral-7B-shaped layer, 8K context", "mha": "MHA-style layer, 128K context",
                           "ragged": "ragged decode batch, 32 sequences, context log-uniform in [1K, 64K]"}
                     .get(wl.name, wl.name)),
        "batch": wl.batch, "q_heads": wl.num_q_heads, "kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
        "context": max(wl.ctx_lens), "page_size": wl.page_size, "prefill_chunk": wl.prefill_chunk,
        "heads": {"global": kinds.get("global", 0), "local": kinds.get("local", 0)},
        "local_sink_window": list(loc) if loc else None,
        "inputs": "i.i.d. N(0,1) bf16, per-rank seed",
        "l2": "flushed before every timed kernel (256 MB write + 512 MB read)",
        "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU",
    }


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def reduce_max(values, world: int, device) -> list[float]:
    """Element-wise max over ranks (the slowest rank sets every timing)."""
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank processed the same units in at most max_ms."""
    return world * units_per_rank / (max_ms * 1e-3)


def kernel_traffic(kernel: str, source: Path, workload_name: str) -> int | None:
    """DRAM bytes per launch from the last ncu capture of this workload, if the kernel source is unchanged since."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    rec = json.loads(p.read_text()).get(kernel)
    if not rec or rec.get("workload_key") != workload_name:
        return None
    sha = hashlib.sha256(source.read_bytes()).hexdigest()[:16]
    return int(rec["bytes_per_launch"]) if rec.get("source_sha16") == sha else None


def median_ms(fn, flush, n: int) -> float:
    """Median CUDA-event time of fn() over n runs, L2 flushed before each (after one untimed run)."""
    import torch
    fn()
    vals = []
    for _ in range(n):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        vals.append(e0.elapsed_time(e1))
    return statistics.median(vals)


def run_ours(args) -> None:
    import torch
    import torch.distributed as dist

    from head_aware_paged_build_b200 import workloads as W
    from head_aware_paged_build_b200.runtime import layer_for
    from head_aware_paged_build_b200 import segpaged as S

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = workload(args.workload, rank)
    # A configuration without a prefill chunk (the ragged decode batch) is decode only:
    # its step is pack + decode, and the decode kernel is its dominant kernel.
    has_pre = wl.prefill_chunk is not None
    dec = wl.decode_problem()
    pre = wl.prefill_problem() if has_pre else None
    k, v = W.dense_kv(dec, device=dev, gen_device=dev)
    qd = W.queries(dec, device=dev, gen_device=dev)
    Ld = layer_for(dec, device=dev)
    od, lsed = torch.empty_like(qd), torch.empty(qd.shape[:2], dtype=torch.float32, device=dev)
    if has_pre:
        qp = W.queries(pre, device=dev, gen_device=dev)
        Lp = layer_for(pre, device=dev)
        op, lsep = torch.empty_like(qp), torch.empty(qp.shape[:2], dtype=torch.float32, device=dev)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(128 << 20, dtype=torch.float32, device=dev)

    def flush():
        flush_w.zero_()
        flush_r.sum()

    calls = [lambda: Ld.build(k, v), lambda: Ld.attention(qd, od, lsed)]
    names = ["pack_decode", "decode"]
    if has_pre:
        calls += [lambda: Lp.build(k, v), lambda: Lp.attention(qp, op, lsep)]
        names += ["pack_prefill", "prefill"]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in calls]

    def step(record: bool):
        for i, c in enumerate(calls):
            flush()
            if record:
                ev[i][0].record()
            c()
            if record:
                ev[i][1].record()

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    for lay in ((Ld, Lp) if has_pre else (Ld,)):
        assert lay.device_status() == 0, "device status word set during warm-up"

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    totals = [0.0] * len(calls)
    wall0 = time.perf_counter()
    for _ in range(args.steps):
        step(True)
        torch.cuda.synchronize()
        for i in range(len(calls)):
            totals[i] += ev[i][0].elapsed_time(ev[i][1])
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = dict(zip(names, reduce_max([x / args.steps for x in totals], world, dev)))

    # ---- dense-plus-mask variant (same kernels, every head stores its whole context) ----
    Ldm = layer_for(dec, device=dev, flags=S.SP_FLAG_DENSE_MASKED)
    Ldm.build(k, v)
    dm = {"decode": median_ms(lambda: Ldm.attention(qd, od, lsed), flush, 10)}
    del Ldm
    if has_pre:
        Lpm = layer_for(pre, device=dev, flags=S.SP_FLAG_DENSE_MASKED)
        Lpm.build(k, v)
        dm["prefill"] = median_ms(lambda: Lpm.attention(qp, op, lsep), flush, 3)
        del Lpm
    dm = dict(zip(dm.keys(), reduce_max(list(dm.values()), world, dev)))

    # ---- E4M3 pages: the same decode on 1-byte pages (per-tensor scales amax / 448) ----
    k_scale = float(k.abs().max()) / 448.0
    v_scale = float(v.abs().max()) / 448.0
    Ld8 = layer_for(dec, device=dev, kv_dtype="e4m3", k_scale=k_scale, v_scale=v_scale)
    Ld8.build(k, v)
    fp8_ms = median_ms(lambda: Ld8.attention(qd, od, lsed), flush, 10)
    fp8_pack_ms = median_ms(lambda: Ld8.build(k, v), flush, 5)
    assert Ld8.device_status() == 0, "device status word set by the E4M3 decode"
    fp8_ms, fp8_pack_ms = reduce_max([fp8_ms, fp8_pack_ms], world, dev)
    del Ld8

    # ---- retrieval heads: the 32K layer with two retrieval kv-heads per sequence ----
    retrieval = run_retrieval(wl, dev, flush, world) if wl.name.startswith("llama") else None

    # ---- end to end through the public API with host buffers ----
    e2e_dense = run_e2e_dense(args, dev, Ld, k, v, qd, od, lsed, world)
    e2e, append_us = run_e2e_serving(args, dev, wl, dec, k, v, world)
    e2e["dense_upload_variant"] = e2e_dense

    zd = Ld.sizes
    zp = Lp.sizes if has_pre else None
    eb = 2
    vis_dec = zd.stored_token_heads * 2 * wl.head_dim * eb          # K + V rows the decode must read
    pack_bytes = lambda z: z.stored_token_heads * 2 * wl.head_dim * eb + 2 * z.num_pages * z.page_bytes
    pk = peaks()
    dec_gbs = weak_rate(vis_dec, world, ms["decode"]) / 1e9
    launches_per_step = 1 + zd.kernel_launches() + ((1 + zp.kernel_launches()) if has_pre else 0)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    csrc = ROOT / "head_aware_paged_build_b200" / "csrc"
    roof_dec = {"kernel": "decode_mma_kernel", "bound": "hbm",
                "achieved": round(vis_dec / (ms["decode"] * 1e-3) / 1e9, 1), "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": round(vis_dec / (ms["decode"] * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                "peak_source": f"{pk['source']} HBM copy",
                "traffic": kernel_traffic("decode_mma_kernel", csrc / "kernels_decode.cu", wl.name)}
    if has_pre:
        flops_pre = 4 * wl.head_dim * zp.visible_pairs              # QK^T + PV on visible pairs
        pre_tflops = weak_rate(flops_pre, world, ms["prefill"]) / 1e12
        per_launch_pre = flops_pre / (ms["prefill"] * 1e-3) / 1e12
        # Each kernel is timed alone (L2 flushes between them), so the burst GEMM figure is
        # the denominator; the sustained one is reported beside it in "prefill".
        pre_peak = pk["bf16_tflops"]
        prefill = {"ms": round(ms["prefill"], 4), "visible_flops": flops_pre, "TFLOP/s": round(pre_tflops, 1),
                   "frac_bf16_burst": round(pre_tflops / world / pk["bf16_tflops"], 4),
                   "frac_bf16_sustained": round(pre_tflops / world / pk["bf16_tflops_sustained"], 4)}
        roof = {"kernel": "prefill_tc_kernel", "bound": "tensor", "achieved": round(per_launch_pre, 1),
                "peak": pre_peak, "unit": "TFLOP/s", "frac": round(per_launch_pre / pre_peak, 4),
                "peak_source": f"{pk['source']} bf16 burst",
                "traffic": kernel_traffic("prefill_tc_kernel", csrc / "kernels_prefill_tc.cu", wl.name)}
    else:
        prefill, roof = None, roof_dec  # decode-only configuration: the decode kernel dominates
    line = {
        "metric": METRIC,
        "value": round(dec_gbs, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(sum(ms.values()), 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(wl, world),
        "decode": {"ms": round(ms["decode"], 5), "visible_kv_bytes": vis_dec, "GB/s": round(dec_gbs, 1),
                   "frac_hbm": round(dec_gbs / world / pk["hbm_gbs"], 4), "launches": zd.kernel_launches()},
        "prefill": prefill,
        "pack": {"decode_ms": round(ms["pack_decode"], 5),
                 "decode_GB/s": round(pack_bytes(zd) / (ms["pack_decode"] * 1e-3) / 1e9, 1),
                 **({"prefill_ms": round(ms["pack_prefill"], 5),
                     "prefill_GB/s": round(pack_bytes(zp) / (ms["pack_prefill"] * 1e-3) / 1e9, 1)} if has_pre else {})},
        "dense_masked": {"decode_ms": round(dm["decode"], 5), "decode_skip": round(dm["decode"] / ms["decode"], 3),
                         **({"prefill_ms": round(dm["prefill"], 4),
                             "prefill_skip": round(dm["prefill"] / ms["prefill"], 3)} if has_pre else {}),
                         "kv_saving": round(1 - zd.stored_token_heads / zd.dense_token_heads, 4)},
        "roofline": roof,
        "roofline_decode": roof_dec,
        "decode_e4m3": {"ms": round(fp8_ms, 5), "visible_kv_bytes": vis_dec // eb,
                        "GB/s": round(weak_rate(vis_dec // eb, world, fp8_ms) / 1e9, 1),
                        "frac_hbm": round(vis_dec // eb / (fp8_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                        "speedup_vs_bf16": round(ms["decode"] / fp8_ms, 3), "pack_ms": round(fp8_pack_ms, 5),
                        "what": "decode on FP8 E4M3 pages (1 byte per element), bf16 queries and output"},
        "e2e": e2e,
        "append": {"us": round(append_us, 2), "what": "segpaged_decode_append: one token per sequence, all heads"},
        "retrieval": retrieval,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "wall_s_timed": round(wall, 3),
    }
    if world == 1 and not args.no_cpu_baseline:
        Ld.attention(qd, od, lsed)  # the measured kernels' outputs, checked on the oracle's samples
        if has_pre:
            Lp.attention(qp, op, lsep)
        torch.cuda.synchronize()
        line["cpu_baseline"] = cpu_baseline(wl, dec, k, v, qd, args.cpu_seconds, gpu=(od, lsed),
                                            pre=pre, qp=qp if has_pre else None,
                                            gpu_pre=(op, lsep) if has_pre else None,
                                            prefill_full=args.cpu_prefill_full)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_retrieval(wl, dev, flush, world) -> dict:
    """Decode and prefill of the 32K layer with retrieval heads (same shape and batch as `wl`).

    Per sequence: the layer's global kv-head, two retrieval kv-heads (sink 4, window 512,
    top_p 0.5 of the synthetic per-page importance) and five local ones (sink 4, window 8192).
    Rates count only the work the heads' visible sets need: stored K+V bytes for decode,
    4 * head_dim FLOPs per visible pair for prefill.  The scoring pass that computes a
    retrieval head's importance (attention mass per page, segpaged_block_mass) is timed on
    the same layer: it reads every key once.
    """
    import torch

    from head_aware_paged_build_b200 import segpaged as S
    from head_aware_paged_build_b200 import workloads as W
    from head_aware_paged_build_b200.runtime import layer_for

    wr = W.llama_retrieval(batch=wl.batch)
    dec, pre = wr.decode_problem(), wr.prefill_problem()
    k, v = W.dense_kv(dec, device=dev, gen_device=dev)
    qd = W.queries(dec, device=dev, gen_device=dev)
    qp = W.queries(pre, device=dev, gen_device=dev)
    ld, lp = layer_for(dec, device=dev), layer_for(pre, device=dev)
    ld.build(k, v)
    lp.build(k, v)
    od, lsed = torch.empty_like(qd), torch.empty(qd.shape[:2], dtype=torch.float32, device=dev)
    op, lsep = torch.empty_like(qp), torch.empty(qp.shape[:2], dtype=torch.float32, device=dev)
    d_ms = median_ms(lambda: ld.attention(qd, od, lsed), flush, 10)
    p_ms = median_ms(lambda: lp.attention(qp, op, lsep), flush, 3)
    assert ld.device_status() == 0 and lp.device_status() == 0
    # the scoring pass that gives retrieval heads their importance (segpaged_block_mass):
    # every key of every (sequence, kv-head) read once, with the queries at the last position
    B, hkv, L, d = k.shape
    mprob = S.make_problem(B, wr.num_q_heads, hkv, d, wr.page_size, "bf16", dec.ctx_lens,
                           [x - 1 for x in dec.ctx_lens], [("global", 0, 0)] * (B * hkv))
    nb = -(-L // wr.page_size)
    mass = torch.empty(B, hkv, nb, dtype=torch.float32, device=dev)
    mws = torch.empty(S.segpaged_block_mass_workspace(mprob), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    m_ms = median_ms(lambda: S.segpaged_block_mass(mprob, k.data_ptr(), k.stride(0), k.stride(1), k.stride(2),
                                                   qd.data_ptr(), 0.0, mass.data_ptr(), nb, mws.data_ptr(),
                                                   mws.numel(), stream), flush, 10)
    d_ms, p_ms, m_ms = reduce_max([d_ms, p_ms, m_ms], world, dev)
    pk = peaks()
    vis = ld.sizes.stored_token_heads * 2 * wr.head_dim * 2
    flops = 4 * wr.head_dim * lp.sizes.visible_pairs
    key_bytes = sum(dec.ctx_lens) * hkv * d * 2
    return {"block_mass_ms": round(m_ms, 5), "block_mass_key_bytes": key_bytes,
            "block_mass_GB/s": round(weak_rate(key_bytes, world, m_ms) / 1e9, 1),
            "block_mass_frac_hbm": round(key_bytes / (m_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
            "decode_ms": round(d_ms, 5), "decode_visible_kv_bytes": vis,
            "decode_GB/s": round(weak_rate(vis, world, d_ms) / 1e9, 1),
            "decode_frac_hbm": round(vis / (d_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
            "prefill_ms": round(p_ms, 4), "prefill_visible_flops": flops,
            "prefill_TFLOP/s": round(weak_rate(flops, world, p_ms) / 1e12, 1),
            "prefill_frac_bf16_burst": round(flops / (p_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
            "kv_saving_decode": round(1 - ld.sizes.stored_token_heads / ld.sizes.dense_token_heads, 4),
            "what": "32K layer, per sequence 1 global, 2 retrieval (sink 4, window 512, top_p 0.5 of synthetic "
                    "per-page importance), 5 local kv-heads"}


def run_e2e_serving(args, dev, wl, dec, k, v, world) -> tuple[dict, float]:
    """Serving decode steps through the public API, cache resident on the GPU.

    A ring plan of the decode layer is built once (untimed).  Every timed step
    copies that step's inputs from pinned host memory (the new token's K and V
    rows and its queries), appends the token and runs decode attention, and
    copies O and LSE back to the host.  The headline replays the step from a
    CUDA graph with segpaged_decode_step (append and attention in one launch);
    the same graph with the two calls (segpaged_decode_append,
    segpaged_attention) and the eager two-call step are reported beside it.
    """
    import torch

    from head_aware_paged_build_b200 import segpaged as S
    from head_aware_paged_build_b200 import workloads as W
    from head_aware_paged_build_b200.runtime import DecodeStepGraph, layer_for

    n_steps = args.warmup + max(3, args.steps // 2)
    start = W.Problem(wl, tuple(L - n_steps for L in dec.ctx_lens), tuple(L - n_steps - 1 for L in dec.ctx_lens))
    layer = layer_for(start, device=dev, flags=S.SP_FLAG_RING, append_capacity=n_steps)
    layer.build(k, v)
    B, Hkv, Hq, d = wl.batch, wl.num_kv_heads, wl.num_q_heads, wl.head_dim
    kin = torch.empty(n_steps, B, Hkv, d, dtype=k.dtype).pin_memory()
    vin = torch.empty_like(kin).pin_memory()
    qin = torch.empty(n_steps, B, Hq, d, dtype=k.dtype).pin_memory()
    for i in range(n_steps):
        pos = [L + i for L in start.ctx_lens]
        kin[i] = torch.stack([k[b, :, p] for b, p in enumerate(pos)]).cpu()
        vin[i] = torch.stack([v[b, :, p] for b, p in enumerate(pos)]).cpu()
        qin[i] = W.queries(W.Problem(wl, tuple(p + 1 for p in pos), tuple(pos)), gen_device=dev).cpu()
    kd, vd = torch.empty(B, Hkv, d, dtype=k.dtype, device=dev), torch.empty(B, Hkv, d, dtype=k.dtype, device=dev)
    qdev = torch.empty(B, Hq, d, dtype=k.dtype, device=dev)
    od = torch.empty_like(qdev)
    lsed = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    lh = torch.empty(lsed.shape, dtype=torch.float32).pin_memory()
    s = torch.cuda.current_stream()
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    times, app = [], []
    for i in range(n_steps):
        e0.record(s)
        kd.copy_(kin[i], non_blocking=True)
        vd.copy_(vin[i], non_blocking=True)
        qdev.copy_(qin[i], non_blocking=True)
        e2.record(s)
        layer.append(kd, vd)
        layer.attention(qdev, od, lsed)
        oh.copy_(od, non_blocking=True)
        lh.copy_(lsed, non_blocking=True)
        e1.record(s)
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    # the append alone, on a second ring plan with its own capacity
    probe = layer_for(start, device=dev, flags=S.SP_FLAG_RING, append_capacity=64)
    probe.build(k, v)
    for i in range(8):
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(s)
        probe.append(kd, vd)
        eb.record(s)
        torch.cuda.synchronize()
        app.append(ea.elapsed_time(eb) * 1e3)
    # the same steps replayed from a CUDA graph on a fresh ring plan: the fused step
    # (segpaged_decode_step, one launch), then the two calls (append, attention)
    def graph_ms(fused: bool) -> float:
        glayer = layer_for(start, device=dev, flags=S.SP_FLAG_RING, append_capacity=n_steps)
        glayer.build(k, v)
        step = DecodeStepGraph(glayer, fused=fused)
        gtimes = []
        for i in range(n_steps):
            step.k_in.copy_(kin[i]), step.v_in.copy_(vin[i]), step.q_in.copy_(qin[i])  # host-side refill
            e0.record(s)
            step.replay()
            e1.record(s)
            torch.cuda.synchronize()
            if i >= args.warmup:
                gtimes.append(e0.elapsed_time(e1))
        assert glayer.device_status() == 0
        del step
        return statistics.median(gtimes)

    g_fused, g_two = graph_ms(True), graph_ms(False)
    assert layer.device_status() == 0 and probe.device_status() == 0
    ms, ms_two, ms_eager = reduce_max([g_fused, g_two, statistics.median(times)], world, dev)
    vis = layer.sizes.stored_token_heads * 2 * d * k.element_size()
    h2d = (kin[0].numel() + vin[0].numel() + qin[0].numel()) * kin.element_size()
    d2h = oh.numel() * oh.element_size() + lh.numel() * 4
    path = ("pinned host q, k_new, v_new -> segpaged_decode_append -> segpaged_attention (decode, cache resident) "
            "-> host O, LSE")
    fused = ("pinned host q, k_new, v_new -> segpaged_decode_step (append + decode attention in one launch, "
             "cache resident) -> host O, LSE, replayed from a CUDA graph")
    two = path + ", replayed from a CUDA graph"
    # the headline is the faster of the two graph-replayed serving steps; the other is reported beside it
    (ms_h, path_h), (ms_o, path_o) = sorted([(ms, fused), (ms_two, two)])
    rec = lambda m, pth: {"value": round(weak_rate(vis, world, m) / 1e9, 2), "unit": "GB/s",
                          "ms_per_step": round(m, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                          "path": pth}
    return ({**rec(ms_h, path_h),
             "other_graph_variant": rec(ms_o, path_o),
             "eager_variant": {"value": round(weak_rate(vis, world, ms_eager) / 1e9, 2), "unit": "GB/s",
                               "ms_per_step": round(ms_eager, 4), "h2d_bytes_per_step": h2d,
                               "d2h_bytes_per_step": d2h, "path": path + ", issued call by call"}},
            statistics.median(app))


def run_e2e_dense(args, dev, layer, k, v, qd, od, lsed, world) -> dict:
    """Decode with the whole dense K/V uploaded from pinned host memory and packed every step."""
    import torch
    kh, vh, qh = (t.cpu().pin_memory() for t in (k, v, qd))
    oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    lh = torch.empty(lsed.shape, dtype=lsed.dtype).pin_memory()
    kd, vd, qdd = torch.empty_like(k), torch.empty_like(v), torch.empty_like(qd)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for i in range(args.warmup + max(3, args.steps // 4)):
        e0.record(s)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        qdd.copy_(qh, non_blocking=True)
        layer.build(kd, vd)
        layer.attention(qdd, od, lsed)
        oh.copy_(od, non_blocking=True)
        lh.copy_(lsed, non_blocking=True)
        e1.record(s)
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    ms = reduce_max([statistics.median(times)], world, dev)[0]
    vis = layer.sizes.stored_token_heads * 2 * k.shape[-1] * k.element_size()
    h2d = (kh.numel() + vh.numel()) * kh.element_size() + qh.numel() * qh.element_size()
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
    return {"value": round(weak_rate(vis, world, ms) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "path": "pinned host K/V/Q -> build_segpaged_cache -> segpaged_attention (decode) -> host O, LSE"}


def host_cores() -> int:
    """Host cores this process may run on (its CPU affinity), the oracle's OpenMP default."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _f64(t):
    return t.double().cpu().numpy()


def _cos(a, r) -> float:
    import numpy as np
    return float(a.ravel() @ r.ravel() / (np.linalg.norm(a) * np.linalg.norm(r)))


def oracle_decode_sample(wl, dec, k, v, qd, budget_s: float, max_groups: int | None = None,
                         gpu: tuple | None = None) -> tuple[float, int, int, dict | None]:
    """Run the CPU oracle on whole (sequence, kv-head) groups until the time budget is spent.

    Groups go to the oracle several at a time in one batched call, so that every host core
    works on their rows (one decode row per q-head).  Returns (seconds spent inside the
    oracle, visible KV bytes covered, groups done, parity), where parity compares the GPU
    decode output `gpu` = (out, lse) with the oracle on the same groups (per q-head cosine and
    max abs error of O, max abs error of LSE), or is None without `gpu`.
    """
    import numpy as np

    import oracle

    spent, vis, done = 0.0, 0, 0
    cos_min, abs_max, lse_max = 1.0, 0.0, 0.0
    if gpu is not None:
        gout, glse = _f64(gpu[0]), _f64(gpu[1])
    order = [(b, kv) for b in range(wl.batch) for kv in range(wl.num_kv_heads)]
    if max_groups is not None:
        order = order[:max_groups]
    per_call = max(1, int(1.5e9 // (2 * max(dec.ctx_lens) * wl.head_dim * 8)))  # <= 1.5 GB of fp64 K/V per call
    for c0 in range(0, len(order), per_call):
        if spent >= budget_s:
            break
        chunk = order[c0:c0 + per_call]
        groups = []
        for b, kv in chunk:
            L = dec.ctx_lens[b]
            kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
            groups.append((_f64(qd[b, kv * wl.group:(kv + 1) * wl.group]), [L - 1] * wl.group,
                           _f64(k[b, kv, :L]), _f64(v[b, kv, :L]), kind, s, w))
        t0 = time.perf_counter()
        res = oracle.attention_batch(groups)
        spent += time.perf_counter() - t0
        for (b, kv), (o_ref, l_ref), gr in zip(chunk, res, groups):
            L = dec.ctx_lens[b]
            vis += int(oracle.stored_mask(gr[4], gr[5], gr[6], L, L - 1).sum()) * 2 * wl.head_dim * 2
            done += 1
            if gpu is not None:
                for i in range(wl.group):
                    a, r = gout[b, kv * wl.group + i], o_ref[i]
                    cos_min = min(cos_min, _cos(a, r))
                    abs_max = max(abs_max, float(np.max(np.abs(a - r))))
                    lse_max = max(lse_max, abs(float(glse[b, kv * wl.group + i]) - float(l_ref[i])))
    parity = ({"min_cos": round(cos_min, 7), "max_abs": float(f"{abs_max:.3g}"), "max_lse_abs": float(f"{lse_max:.3g}"),
               "heads": done * wl.group, "against": "fp64 oracle, same inputs"} if gpu is not None else None)
    return spent, vis, done, parity


def oracle_prefill_sample(wl, pre, k, v, qp, budget_s: float, full: bool = False, rows_per_head: int = 48,
                          gpu: tuple | None = None) -> dict:
    """The CPU oracle on the prefill chunk: visible-pair FLOPs per second of host time.

    Groups (sequence, kv-head) are taken in a seeded random order; from each, `rows_per_head`
    seeded random rows of every q-head of the group (all rows with `full`), several groups per
    batched oracle call, until the time budget is spent (or, with `full`, every row is done).
    The rate counts 4 * head_dim FLOPs per visible (query, key) pair, as the GPU prefill's;
    the time of the whole chunk is that work divided by the rate (extrapolated unless `full`).
    With `gpu` = (out, lse) of the GPU prefill the same rows are compared with the oracle.
    """
    import numpy as np

    import oracle

    rng = np.random.default_rng(12345)
    order = [(b, kv) for b in range(wl.batch) for kv in range(wl.num_kv_heads)]
    order = [order[i] for i in rng.permutation(len(order))]
    off = pre.q_offsets
    per_call = max(1, int(1.5e9 // (2 * max(pre.ctx_lens) * wl.head_dim * 8)))
    spent, pairs, rows_done, done = 0.0, 0, 0, 0
    cos_min, abs_max, lse_max = 1.0, 0.0, 0.0
    if gpu is not None:
        gout, glse = gpu
    for c0 in range(0, len(order), per_call):
        if spent >= budget_s and not full:
            break
        chunk = order[c0:c0 + per_call]
        groups, meta = [], []
        for b, kv in chunk:
            L, q0 = pre.ctx_lens[b], pre.q_starts[b]
            C = L - q0
            kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
            rows = np.arange(C) if full else np.sort(rng.choice(C, min(C, rows_per_head), replace=False))
            kk, vv = _f64(k[b, kv, :L]), _f64(v[b, kv, :L])
            for h in range(kv * wl.group, (kv + 1) * wl.group):
                idx = torch_index(off[b] + rows, qp.device)
                groups.append((_f64(qp[idx, h]), q0 + rows, kk, vv, kind, s, w))
                meta.append((b, h, rows, kind, s, w))
        t0 = time.perf_counter()
        res = oracle.attention_batch(groups)
        spent += time.perf_counter() - t0
        done += len(chunk)
        for (b, h, rows, kind, s, w), (o_ref, l_ref) in zip(meta, res):
            q0 = pre.q_starts[b]
            pos = q0 + rows
            if kind == "local":  # |visible(p)| = min(p + 1, s + w); global: p + 1
                pairs += int(np.minimum(pos + 1, s + w).sum())
            else:
                pairs += int((pos + 1).sum())
            rows_done += len(rows)
            if gpu is not None:
                idx = torch_index(off[b] + rows, gout.device)
                a = _f64(gout[idx, h])
                cos_min = min(cos_min, _cos(a, o_ref))
                abs_max = max(abs_max, float(np.max(np.abs(a - o_ref))))
                lse_max = max(lse_max, float(np.max(np.abs(_f64(glse[idx, h]) - l_ref))))
    flops = 4 * wl.head_dim * pairs
    total_rows = pre.total_queries * wl.num_q_heads
    rate = flops / spent
    return {"value": round(rate / 1e12, 6), "unit": "TFLOP/s", "cores": host_cores(),
            "threads": oracle.num_threads(), "kind": "oracle", "seconds": round(spent, 2),
            "extrapolated": not (full and rows_done == total_rows),
            "chunk_s_at_this_rate": round(4 * wl.head_dim * pre_visible_pairs(wl, pre) / rate, 1),
            "sample": (f"prefill rows: {rows_done} of {total_rows} (query row, q-head) pairs, "
                       + ("all rows" if full else f"{rows_per_head} seeded random rows of every q-head")
                       + f" of {done} of {len(order)} (sequence, kv-head) groups in seeded random order; "
                         "rate = 4 * head_dim * visible pairs / oracle time (fp64 dense attention with "
                         "explicit mask)"),
            **({"parity": {"min_cos": round(cos_min, 7), "max_abs": float(f"{abs_max:.3g}"),
                           "max_lse_abs": float(f"{lse_max:.3g}"), "rows": rows_done,
                           "against": "fp64 oracle, same inputs"}} if gpu is not None else {})}


def torch_index(rows, device):
    import torch
    return torch.as_tensor(rows, dtype=torch.long, device=device)


def pre_visible_pairs(wl, pre) -> int:
    """Visible (query, key) pairs of the whole chunk over all q-heads (global p + 1, local min(p + 1, s + w))."""
    n = 0
    for b, (L, q0) in enumerate(zip(pre.ctx_lens, pre.q_starts)):
        for kv in range(wl.num_kv_heads):
            kind, s, w = wl.policy[b * wl.num_kv_heads + kv]
            for p in range(q0, L):
                n += min(p + 1, s + w) if kind == "local" else p + 1
    return n * wl.group


def cpu_baseline(wl, dec, k, v, qd, budget_s: float, gpu: tuple | None = None, pre=None, qp=None,
                 gpu_pre: tuple | None = None, prefill_full: bool = False) -> dict:
    import oracle
    spent, vis, groups, parity = oracle_decode_sample(wl, dec, k, v, qd, budget_s, gpu=gpu)
    out = {"value": round(vis / spent / 1e9, 4), "unit": "GB/s", "cores": host_cores(),
           "threads": oracle.num_threads(), "kind": "oracle",
           "seconds": round(spent, 2),
           "decode_parity": parity,
           "sample": f"decode of {groups} of {wl.batch * wl.num_kv_heads} (sequence, kv-head) groups, "
                     f"all {wl.group} q-heads each, several groups per batched call on all host cores "
                     "(fp64 dense attention with explicit mask)"}
    if pre is not None:
        out["prefill"] = oracle_prefill_sample(wl, pre, k, v, qp, budget_s, full=prefill_full, gpu=gpu_pre)
    return out


def run_reference(args) -> None:
    """The oracle as the reference arm: decode visible-KV GB/s of the fp64 CPU oracle."""
    import torch

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from head_aware_paged_build_b200 import workloads as W

    wl = workload(args.workload, 0)
    dec = wl.decode_problem()
    # inputs on the host (CPU generator): the oracle never touches the GPU
    k, v = W.dense_kv(dec)
    qd = W.queries(dec)
    per_step = max(1, wl.num_kv_heads // 2)
    for _ in range(args.warmup):
        oracle_decode_sample(wl, dec, k, v, qd, 1e9, max_groups=1)
    spent = vis = 0.0
    for _ in range(args.steps):
        s, b, _, _ = oracle_decode_sample(wl, dec, k, v, qd, 1e9, max_groups=per_step)
        spent += s
        vis += b
    value = vis / spent / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * spent / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, 1),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": host_cores(),
                         "threads": oracle.num_threads(), "kind": "oracle",
                         "sample": f"per step: decode of {per_step} (sequence, kv-head) groups of sequence 0 "
                                   f"(all {wl.group} q-heads each) in one batched call on all host cores, "
                                   "fp64 dense attention with explicit mask"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="llama", choices=("llama", "mistral", "mha", "ragged", "llama_b1"))
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="time budget of the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-prefill-full", action="store_true",
                    help="run the oracle over every prefill row (Mistral-sized layers) instead of a sample")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
