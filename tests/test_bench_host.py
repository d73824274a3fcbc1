"""Host logic of the multi-GPU benchmark (replicas), on the CPU with two gloo ranks.

The path shards by sequence with no exchange step, so ``bench.py --gpus N`` runs
N replicas; the only cross-rank steps are a barrier and the max over ranks of
the device times. These tests run exactly those helpers in two processes.
"""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, local_ms: list, q) -> None:
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(local_ms[rank], world)
        value, ms = bench.job_throughput(64 * 10, local_ms[rank], world)
        bench.barrier(world)
        q.put((rank, m, value, ms))
    finally:
        dist.destroy_process_group()


def _run(world: int, local_ms: list) -> list:
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_max_over_ranks_two_gloo_ranks():
    out = _run(2, [12.5, 20.0])
    for rank, m, value, ms in out:
        assert m == 20.0 and ms == 20.0
        # 2 ranks x 640 units over the slowest rank's 20 ms
        assert value == pytest.approx(2 * 640 / 0.020)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    value, ms = bench.job_throughput(100, 50.0, 1)
    assert ms == 50.0 and value == pytest.approx(2000.0)


def test_reference_arm_other_ranks_do_no_work(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup, gpus = 1, 0, 2
    assert bench.run_reference(A(), 2, 1) is None
    assert capsys.readouterr().out == ""
