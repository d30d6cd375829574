"""The multi-process host logic of bench.py on CPU: two gloo ranks set up
through the same environment variables torchrun provides, the max-over-ranks
time reduction and the whole-job throughput aggregation."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    d = bench.Dist(world)
    try:
        d.barrier()
        seconds = 1.0 + rank            # rank 1 is the slow one
        mx = d.max(seconds)
        value = bench.aggregate(100.0, d.world, mx)
        q.put((rank, d.world, mx, value))
    finally:
        d.close()


def test_two_gloo_ranks_reduce_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, world, mx, value in res:
        assert world == 2
        assert mx == 2.0               # the slowest rank's time
        assert value == 100.0          # 2 ranks x 100 units / 2 s


def test_single_process_without_torchrun():
    import bench
    os.environ.pop("WORLD_SIZE", None)
    d = bench.Dist(1)
    assert d.world == 1 and d.max(3.5) == 3.5
    assert bench.aggregate(10.0, 1, 2.0) == 5.0
