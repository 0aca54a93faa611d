"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2).

DSA shards with no collective on its data path: every rank runs the same
workload on its own seeded inputs, and only the timing is reduced (max over
ranks).  These tests run that host logic in two gloo processes."""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _worker(rank: int, world: int, store_file: str, results):
    import datetime
    # a file rendezvous: no port to race for
    dist.init_process_group("gloo", init_method=f"file://{store_file}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from sparse_attention_weight_b200 import inputs
        from sparse_attention_weight_b200.configs import Workload
        # timing: each rank reports its own elapsed time; everyone gets the max
        mine = 10.0 + 5.0 * rank
        got = bench.reduce_max(mine)
        # shards: same shapes, different data per rank
        wl = Workload("mr", 60, "decode", k=64, h_index=8, heads=8, batch=3, ctx_min=50, ctx_max=90, q_per_seq=2)
        ins = inputs.make_inputs(wl, seed=bench.rank_seed(rank))
        digest = float(ins["w"].astype(np.float64).sum())
        shapes = {k: v.shape for k, v in ins.items() if hasattr(v, "shape")}
        t = torch.tensor([digest], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, t)
        results[rank] = (got, shapes, [float(g.item()) for g in gathered], ins["batch"].num_q)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_timing_and_draw_distinct_shards(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    store = str(tmp_path / "rendezvous")
    procs = [ctx.Process(target=_worker, args=(r, world, store, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == 15.0                      # max over ranks
    assert r0[1] == r1[1]                              # same per-rank workload shape
    assert r0[2] == r1[2] and r0[2][0] != r0[2][1]     # different seeded data per rank
    import bench
    assert bench.whole_job_rate(r0[3], world, 15.0) == pytest.approx(r0[3] * 2 / 0.015)


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
