"""The multi-GPU path of the benchmark is replicas (every (batch, head) is
independent; there is no exchange step): each rank runs the whole layer and
the job is timed by its slowest rank.  This covers that host-side logic with
two gloo ranks on the CPU."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q) -> None:
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    slowest = bench.max_over_ranks(10.0 + 5.0 * rank)  # per-rank "milliseconds"
    dist.barrier()
    q.put((rank, slowest, bench.job_tflops(1e12, 4, world, slowest)))
    dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in results] == [15.0, 15.0]
    # 2 ranks x 4 steps x 1 TFLOP in 15 ms
    assert results[0][2] == pytest.approx(2 * 4 * 1.0 / 15e-3)


def test_single_process_is_its_own_maximum():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_tflops(2e12, 3, 1, 6.0) == pytest.approx(1000.0)
