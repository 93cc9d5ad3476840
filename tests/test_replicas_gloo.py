"""The N > 1 path of bench.py on CPU: two gloo ranks.  The HSA step runs on one
GPU, so bench.py runs independent replicas with no data-path collective; the
only cross-rank step is the max-over-ranks reduction of the timed region and
the barriers around it.  This test runs that host logic with world_size 2."""

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    bench.barrier(dist)
    total_ms = 100.0 + 50.0 * rank                 # rank 1 is the slow one
    got = bench.max_over_ranks(total_ms, dist, "cpu")
    bench.barrier(dist)
    out.put((rank, got))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_over_ranks():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 150.0, 1: 150.0}


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(12.5, None, "cpu") == 12.5
    bench.barrier(None)
