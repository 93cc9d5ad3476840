"""Host logic of the sequence-sharded step, on CPU.

The sharded step splits the active list A_i of an iteration into G chunks and
exchanges, per layer, the fresh K|V rows of every chunk (an all-gather) and,
per step, the fresh velocities (an all-reduce of a buffer that is zero outside
each rank's rows).  These tests run that exchange protocol with stand-in
rows whose values name the A_i position they belong to: through the
in-process driver, and through gloo collectives with world sizes 2 and 3.
The kernels themselves are covered by the GPU tests.
"""

import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from token_sparse_denoising_layer_b200.shard import (  # noqa: E402
    chunk_rows, run_dist, run_local, shard_slices)


@pytest.mark.parametrize("G", [1, 2, 3, 4, 7])
def test_slices_cover_the_active_list_in_order(G):
    for a in range(0, 60):
        c, sl = shard_slices(a, G)
        need = -(-a // G)
        assert c % 4 == 0 and need <= c < max(need, 1) + 4   # 16-byte aligned starts
        assert all(s % 4 == 0 for s, n in sl if n > 0)
        pos = [p for s, n in sl for p in range(s, s + n)]
        assert pos == list(range(a))
        # the all-gather of c-row chunks: its first a rows are A_i's positions in order
        gathered = []
        for s, n in sl:
            gathered += list(range(s, s + n)) + [-1] * (c - n)
        assert gathered[:a] == list(range(a))
        # only trailing chunks are short
        counts = [n for _, n in sl]
        full = [n == c for n in counts]
        assert full == sorted(full, reverse=True) or a == 0
        assert sum(1 for n in counts if 0 < n < c) <= 1


def test_bad_arguments():
    with pytest.raises(ValueError):
        shard_slices(5, 0)
    with pytest.raises(ValueError):
        shard_slices(-1, 2)


def _fake_steps(rank, G, N, D, plan, log):
    """Stand-in for ShardRank.steps: per iteration an active list A (ascending),
    two layers of K|V exchange and one velocity reduction."""
    recv = torch.full((G * chunk_rows(N, G), 2 * D), -7.0)
    send = torch.empty((chunk_rows(N, G), 2 * D))
    v = torch.zeros((N, 4))
    for A in plan:
        a = len(A)
        c, sl = shard_slices(a, G)
        s0, nr = sl[rank]
        for layer in range(2):
            send[:c].fill_(-1.0)                          # padding rows
            send[:nr] = torch.arange(s0, s0 + nr, dtype=torch.float32)[:, None] + 1000 * layer
            yield ("all_gather", send[:c], recv[:G * c])
            got = recv[:a, 0].numpy()
            log.append(bool(np.array_equal(got, np.arange(a) + 1000 * layer)))
            log.append(bool((recv[:a] == recv[:a, :1]).all()))
        v.zero_()
        for p in range(s0, s0 + nr):
            v[A[p]] = float(p + 1)
        yield ("all_reduce_sum", v)
        want = torch.zeros((N, 4))
        for p, t in enumerate(A):
            want[t] = float(p + 1)
        log.append(bool(torch.equal(v, want)))


def _fake_fused_steps(rank, G, N, D, plan, caches, log):
    """Stand-in for ShardRank.steps with the fused K|V exchange: the rank
    writes its chunk's rows straight into every rank's copy of the layer's
    cache (caches[layer, g] is rank g's copy), waits at the barrier, then
    reads its own copy; one velocity reduction per iteration.  The next
    layer writes other buffers, and the next iteration's writes come after
    the reduction, which every rank reaches only after its reads."""
    v = torch.zeros((N, 4))
    sync = torch.zeros((1,), dtype=torch.int32)
    for it, A in enumerate(plan):
        a = len(A)
        _, sl = shard_slices(a, G)
        s0, nr = sl[rank]
        for layer in range(2):
            tag = 1000 * layer + 100000 * it
            for g in range(G):
                for p in range(s0, s0 + nr):
                    caches[layer, g, A[p]] = float(p + tag)
            yield ("barrier", sync)
            got = caches[layer, rank, A, 0].numpy()
            log.append(bool(np.array_equal(got, np.arange(a) + tag)))
            log.append(bool((caches[layer, rank, A] == caches[layer, rank, A, :1]).all()))
        v.zero_()
        for p in range(s0, s0 + nr):
            v[A[p]] = float(p + 1)
        yield ("all_reduce_sum", v)


def _plan(N, seed):
    r = np.random.default_rng(seed)
    sizes = [N, 1, 2, 3, N // 3, 5, N - 1]
    return [np.sort(r.choice(N, size=s, replace=False)).tolist() for s in sizes]


@pytest.mark.parametrize("G", [1, 2, 3])
def test_local_driver_exchanges(G):
    N, D = 37, 4
    logs = [[] for _ in range(G)]
    plan = _plan(N, 3)
    run_local([_fake_steps(r, G, N, D, plan, logs[r]) for r in range(G)])
    for lg in logs:
        assert lg and all(lg)


@pytest.mark.parametrize("G", [1, 2, 3])
def test_local_driver_fused_exchange(G):
    N, D = 37, 4
    logs = [[] for _ in range(G)]
    caches = torch.full((2, G, N, D), -7.0)
    run_local([_fake_fused_steps(r, G, N, D, _plan(N, 3), caches, logs[r]) for r in range(G)])
    for lg in logs:
        assert lg and all(lg)


def test_local_driver_rejects_diverged_ranks():
    def a():
        yield ("all_reduce_sum", torch.zeros(2))

    def b():
        yield ("all_gather", torch.zeros(1, 2), torch.zeros(2, 2))

    with pytest.raises(RuntimeError):
        run_local([a(), b()])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out, caches):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from token_sparse_denoising_layer_b200.shard import run_dist as rd

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    log = []
    rd(_fake_steps(rank, world, 37, 4, _plan(37, 3), log))
    # the fused exchange: every rank writes into all copies held in shared memory
    rd(_fake_fused_steps(rank, world, 37, 4, _plan(37, 3), caches, log))
    dist.barrier()
    out.put((rank, len(log), all(log)))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_exchange(world):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    caches = torch.full((2, world, 37, 4), -7.0).share_memory_()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, caches))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [q.get(timeout=10) for _ in range(world)]
    assert sorted(r for r, _, _ in res) == list(range(world))
    assert all(n > 0 and ok for _, n, ok in res)


def test_dist_driver_rejects_unknown_request():
    def bad():
        yield ("broadcast", torch.zeros(1))

    with pytest.raises(ValueError):
        run_dist(bad())
