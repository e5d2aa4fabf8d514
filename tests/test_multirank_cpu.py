"""The N > 1 path of the benchmark on CPU: independent replicas, the step time
reduced with MAX over ranks, whole-job tokens/s = all ranks' tokens over the
slowest rank's time.  Two gloo ranks on 127.0.0.1; no GPU involved."""
from __future__ import annotations

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow replica
        mx = bench.max_over_ranks(ms, "cpu", world)
        out[rank] = (mx, bench.aggregate_tokens_per_s(world, 131072, mx))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for pr in procs:
            pr.start()
        for pr in procs:
            pr.join(timeout=120)
            assert pr.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == pytest.approx(15.0)
    # 2 x 131072 tokens in 15 ms
    assert res[0][1] == pytest.approx(2 * 131072 / 0.015)


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(3.5, "cpu", 1) == 3.5
    assert bench.aggregate_tokens_per_s(1, 1000, 1.0) == pytest.approx(1e6)
