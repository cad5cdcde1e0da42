"""The N > 1 host path of bench.py on CPU: world size 2 over gloo.  Each rank runs
its own replica; the only collectives are a barrier and a max of the timings."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        bench.barrier(world)
        mine = 1.0 + rank * 0.5  # rank 1 is the slower one
        slowest = bench.max_over_ranks(mine, world, torch.device("cpu"))
        q.put((rank, slowest, bench.whole_job_value(10**12, 2.0, world)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [1.5, 1.5]  # both ranks report the max
    assert got[0][2] == pytest.approx(2 * 10**12 / 2e-3 / 1e12)  # work of both replicas
