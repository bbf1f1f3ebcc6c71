"""CPU, two processes over gloo: the host logic of the multi-GPU benchmark
path. Every rank runs its own problem (weak scaling); the step time is the
slowest rank's, taken with a MAX all-reduce that every rank joins, and the
job's throughput counts all ranks' work over that time."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = 10.0 + 5.0 * rank                  # rank 1 is the slower one
        got = bench.max_over_ranks(ms, world)
        q.put((rank, got, bench.job_tflops(world, 1.0e12, got)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_slowest_time_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in results] == [0, 1]
    for _, got, tflops in results:
        assert got == 15.0                        # both ranks see the slowest rank's time
        assert tflops == pytest.approx(2 * 1.0e12 / 15e-3 / 1e12)


def test_single_rank_is_its_own_time():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_tflops(1, 4.0e12, 2.0) == pytest.approx(2000.0)
