"""The benchmark's N > 1 plumbing on CPU: two gloo ranks (one process each,
as under torchrun) take the barrier, agree on the slowest rank's time and
report the whole-job rate from it."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = 100.0 + 50.0 * rank          # rank 1 is the slow one
        worst = bench.max_over_ranks(world, ms)
        value = bench.job_throughput(world, 4096, 10, worst)
        bench.barrier(world)
        q.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, worst, value in got:
        assert worst == 150.0
        # 2 ranks x 4096 tokens x 10 steps in 150 ms
        assert abs(value - 2 * 4096 * 10 / 0.150) < 1e-6 * value


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1, 3.5) == 3.5
    assert bench.job_throughput(1, 4096, 200, 125.0) == 4096 * 200 / 0.125
