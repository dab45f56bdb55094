"""The multi-process path of bench.py on CPU (world size 2, gloo): every rank
runs its own replica, the job's time is the slowest rank's, and the value is
all ranks' units over that time (weak scaling, no collective on the data path)."""
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    my_ms = 100.0 + 50.0 * rank            # rank 1 is the slow one
    bench._barrier(dist)
    worst = bench._max_over_ranks(my_ms, dist, device="cpu")
    value = bench.weak_scaling_value(1e9, world, worst)
    out.put((rank, worst, value))
    dist.destroy_process_group()


def test_two_rank_max_and_weak_value():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [150.0, 150.0]          # both ranks see the max
    assert res[0][2] == pytest.approx(2 * 1e9 / 0.150)    # all units / slowest time


def test_single_rank_value():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench._max_over_ranks(3.0, None) == 3.0
    assert bench.weak_scaling_value(2e9, 1, 1000.0) == pytest.approx(2e9)
