"""The multi-GPU path of bench.py is replicas only: every rank runs the same
step on its own GPU and the job's time is the slowest rank's.  These tests run
that aggregation on two gloo ranks on the CPU (no GPU, no NCCL)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ms = bench.replicas_time(times[rank], world, torch.device("cpu"))
        out[rank] = (ms, bench.replicas_value(ms, world, 10, 1_000_000))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(2.0, 3.5), (4.0, 1.0)])
def test_replicas_max_over_ranks_gloo(times):
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, list(times), out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    want = max(times)
    for r in range(world):
        ms, value = out[r]
        assert ms == pytest.approx(want)
        # 2 ranks x 10 steps x 1 MB in the slowest rank's time
        assert value == pytest.approx(2 * 10 * 1_000_000 / (want * 1e-3) / 1e9)




def test_single_rank_is_local_time():
    import bench

    assert bench.replicas_time(7.5, 1, torch.device("cpu")) == 7.5
    assert bench.replicas_value(2.0, 1, 4, 1_000_000) == pytest.approx(2.0)
