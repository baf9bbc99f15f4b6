"""The multi-rank logic of bench.py on CPU: two gloo ranks, each with its own
device time, agree on the max over ranks and on the whole-job value (both
replicas' bytes over the slowest rank's time).  The GPU path runs the same
functions with NCCL."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank              # rank 1 is the slower replica
        total = bench.max_over_ranks(mine, world, torch.device("cpu"))
        value = bench.whole_job_gbs(world, 4, 1e9, total)
        dist.barrier()
        q.put((rank, total, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, total, value in got:
        assert total == 15.0
        assert abs(value - 2 * 4 * 1e9 / 15e-3 / 1e9) < 1e-9


def test_single_rank_value_is_its_own():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert abs(bench.whole_job_gbs(1, 10, 2e6, 4.0) - 10 * 2e6 / 4e-3 / 1e9) < 1e-12
