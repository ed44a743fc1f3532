"""bench.py's multi-rank plumbing on CPU: two gloo ranks (127.0.0.1) run the timing
reduction the GPU job uses -- the barrier, the max over ranks of each rank's device time,
and the weak-scaling aggregate (every rank's units over the slowest rank's time)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        my_ms = [12.5, 20.0][rank]                       # rank 1 is the slowest
        worst = bench.max_over_ranks(my_ms, world)
        value = bench.weak_scaling_value(1e12, world, worst, steps=10)
        q.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, value in res:
        assert worst == 20.0
        # 2 ranks x 1e12 units per step, 2.0 ms per step (20 ms / 10 steps)
        assert value == pytest.approx(2e12 / 2e-3)


def test_single_rank_needs_no_collective():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.weak_scaling_value(10.0, 1, 5.0, 5) == pytest.approx(10.0 / 1e-3)
