"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The path shards into independent batches, one per rank: no data-path
collective.  What the ranks share is checked here without a GPU: per-rank
workloads differ only in their seed, every rank plans the same layout, and
timings reduce to the max over ranks with whole-job throughput computed from
it.
"""
from __future__ import annotations

import os
import sys
from pathlib import Path

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _worker(rank: int, world: int, port: int, q) -> None:
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from head_aware_paged_build_b200 import segpaged as S

        wl = bench.workload("mistral", rank)
        prob = wl.decode_problem()
        p = S.make_problem(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.page_size, wl.dtype,
                           prob.ctx_lens, prob.q_starts, wl.policy)
        plan = S.segpaged_plan_create(p)
        z = S.segpaged_plan_sizes(plan).as_dict()
        S.segpaged_plan_destroy(plan)
        # rank r pretends its kernels took (1 + r) ms and (10 - r) ms
        mx = bench.reduce_max([1.0 + rank, 10.0 - rank], world, torch.device("cpu"))
        rate = bench.weak_rate(z["stored_token_heads"], world, mx[0])
        gathered = [None] * world
        dist.all_gather_object(gathered, (wl.seed, z, mx, rate))
        q.put((rank, gathered))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_independent_batches():
    from head_aware_paged_build_b200 import build_ext
    build_ext.build()
    world, port = 2, 29511 + os.getpid() % 1000
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    g = results[0]
    assert results[1] == g
    seeds = [x[0] for x in g]
    assert len(set(seeds)) == world                    # each rank draws its own batch
    assert g[0][1] == g[1][1]                          # ... with the same layout
    assert g[0][2] == g[1][2] == [2.0, 10.0]           # max over ranks, element-wise
    stored = g[0][1]["stored_token_heads"]
    assert g[0][3] == pytest.approx(world * stored / 2.0e-3)
