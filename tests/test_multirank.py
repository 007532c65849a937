"""The multi-rank host path of bench.py on CPU: two gloo ranks.

Each rank runs its own independently seeded problem of the same shapes (the
path shards by (batch, head) problems with no exchange), the step time is the
maximum over ranks, and the reported value aggregates all ranks' work."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from block_sparse_approximate_b200 import workloads as wl
        w = wl.WORKLOADS["video_dit"]
        wr = bench.rank_workload(w, rank)
        inp = wl.prefill_inputs(wr, "cpu", H=1, N=2 * 64 * 64)
        ms = bench._max_over_ranks(1.0 + rank, world, device="cpu")
        bench._barrier(world)
        out[rank] = (wr.seed, ms, float(inp["Q"].float().sum()), bench.job_value(w, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=False)
    import time
    deadline = time.time() + 240
    while not ctx.join(timeout=5):      # join returns once per exiting rank
        if time.time() > deadline:
            for p in ctx.processes:
                p.kill()
            pytest.fail("ranks did not finish")
    seeds = [out[r][0] for r in range(world)]
    assert seeds[0] != seeds[1]                           # independent problems
    assert out[0][2] != out[1][2]                         # ... with different inputs
    assert out[0][1] == out[1][1] == 2.0                  # max over ranks, the same on every rank
    import bench
    from block_sparse_approximate_b200 import workloads as wl
    w = wl.WORKLOADS["video_dit"]
    assert out[0][3] == pytest.approx(2 * bench.dense_flops(w) / 2.0e-3 / 1e12)   # whole-job value
