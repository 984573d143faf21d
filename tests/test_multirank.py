"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

Each rank decodes its own independent batch (weak scaling, no collective on the
data path); the only cross-rank steps are the barrier around the timed region
and the max over ranks of the device time, which these tests exercise."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)     # rank 1 is the slower one
        v = bench.weak_scaling_value(1_000_000_000, world, t, 10)
        bench.barrier(world)
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, t, v in res:
        assert t == 15.0                       # every rank sees the slowest rank's time
        assert v == pytest.approx(2e9 / 1.5e-3 / 1e9)   # 2 ranks x 1 GB per 1.5 ms step


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(2_415_919_104, 1, 425.0, 1000) == pytest.approx(5684.5, rel=1e-3)
