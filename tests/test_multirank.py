"""CPU, two processes over gloo: the host logic of the multi-GPU benchmark
path. Every rank runs its own problem (weak scaling); the step time is the
slowest rank's, taken with a MAX all-reduce that every rank joins, and the
job's throughput counts all ranks' work over that time. For one problem split
by heads, the ranks' head ranges tile the problem and each shard's k-means
seed indices are the whole problem's."""
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


def _split_worker(rank, world, port, q, H, B):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from bit_fp8_attention_prep_b200 import vc_attn
        h0, h1 = vc_attn.head_range(H, rank, world)
        # the seed index of local slice (b, hl) of this shard: b * H + h0 + hl
        mine = [vc_attn.seed_slice_index(b, h0 + hl, H) for b in range(B) for hl in range(h1 - h0)]
        got = [None] * world
        dist.all_gather_object(got, (h0, h1, mine))
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("H,B", [(56, 1), (7, 3)])
def test_head_split_tiles_the_problem_and_keeps_the_seeds(H, B):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q, H, B)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, got in results:
        ranges = [(h0, h1) for h0, h1, _ in got]
        assert ranges[0][0] == 0 and ranges[-1][1] == H and ranges[0][1] == ranges[1][0]   # contiguous, in order
        assert abs((ranges[0][1] - ranges[0][0]) - (ranges[1][1] - ranges[1][0])) <= 1
        seeds = sorted(i for _, _, mine in got for i in mine)
        assert seeds == list(range(B * H))    # every slice of the whole problem once, with its own index


def test_head_slice_of_both_layouts():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    x4 = torch.arange(2 * 3 * 5 * 4).reshape(2, 3, 5, 4)
    assert torch.equal(bench.head_slice(x4, 1, 3), x4[:, :, 1:3]) and bench.head_slice(x4, 1, 3).is_contiguous()
    x3 = x4[0]
    assert torch.equal(bench.head_slice(x3, 2, 5), x3[:, 2:5])
