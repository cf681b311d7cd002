"""Host logic of bench.py's multi-GPU runs (independent replicas), exercised
with world size 2 over gloo on the CPU: every rank gets the slowest rank's
time, and the reported value counts every rank's bytes."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local_ms = [3.0, 5.0][rank]
        slowest = bench.max_over_ranks(local_ms, world)
        bench.barrier(world)
        out[rank] = (slowest, bench.whole_job_gbs(1_000_000, world, slowest))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_bytes():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        slowest, gbs = out[r]
        assert slowest == 5.0
        assert gbs == pytest.approx(2 * 1_000_000 / 5e-3 / 1e9)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.whole_job_gbs(2_000_000_000, 1, 1.0) == pytest.approx(2000.0)
