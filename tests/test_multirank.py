"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, each with its own
batch, a maximum-over-ranks timing reduction and the whole-job aggregate.
(The data path has no collective: replicas only.)"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


PORT = _free_port()


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        class A:
            workload = "tiny"
            B = None
            k = None
            sigma = 1.0
        kind, x, cfg = bench.make_workload(A, rank)
        rows, _ = bench.rows_and_bytes(kind, x)
        # per-rank "times": rank r took 10 + r ms in total, 1 + r ms per call
        mx = bench.reduce_max([10.0 + rank, 1.0 + rank], dist, torch.device("cpu"))
        dist.barrier()
        out[rank] = dict(rows=rows, mx=mx, first=float(x.target.flatten()[0]),
                         value=bench.job_value(rows, world, 5, mx[0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_by_the_slowest_and_count_every_row():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, PORT, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    assert res[0]["mx"] == res[1]["mx"] == [11.0, 2.0]
    assert res[0]["rows"] == res[1]["rows"] == 16
    # each replica verifies its own batch
    assert res[0]["first"] != res[1]["first"]
    # whole-job value: rows of both ranks over the slowest rank's time
    assert res[0]["value"] == pytest.approx(16 * 2 * 5 / 11e-3)


def test_single_rank_helpers_need_no_process_group():
    import bench
    assert bench.reduce_max([1.5, 2.5], None, None) == [1.5, 2.5]
    assert bench.job_value(10, 1, 4, 2.0) == pytest.approx(10 * 4 / 2e-3)
    assert bench.rank_seed(0) != bench.rank_seed(1)
    assert np.isfinite(bench.job_value(1, 8, 1, 1.0))
