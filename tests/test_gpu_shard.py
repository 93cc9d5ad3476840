"""GPU parity of the sequence-sharded step (one loop split over G ranks).

Ranks are emulated in one process on one GPU (their exchanges are device
copies between their buffers, and no kernel waits on another rank), and a
world of one runs through torch.distributed with NCCL.  Every rank must end
with the same latent bit for bit (the replicated parts are deterministic);
the result must match the unsharded loop and the float64 oracle.
"""

import datetime
import os
import socket

import numpy as np
import pytest

from gpu_util import BF16_TOL, bf, dev, host, need_gpu, normwise, torch
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import abi, synth

pytestmark = pytest.mark.gpu


def test_kv_scatter_packed_is_an_exact_copy():
    need_gpu()
    N, D, a = 700, 256, 333
    ctx = abi.hsa_create(N=N, D=D, H=2, F=64, L=1, T=1, budgets=[1], counts=[N])
    ks, vs = synth.stale_kv(N, D, 31)
    idx = synth.random_active_set(N, a, 31)
    kv = synth.bf16_round(synth.rng(32).standard_normal((a, 2 * D), dtype=np.float32))
    kc, vc = bf(ks), bf(vs)
    abi.hsa_kv_scatter_packed(ctx, bf(kv), dev(idx), a, kc, vc)
    abi.hsa_sync_check(ctx)
    want_k, want_v = ks.copy(), vs.copy()
    want_k[idx] = kv[:, :D]
    want_v[idx] = kv[:, D:]
    assert (host(kc) == want_k).all() and (host(vc) == want_v).all()
    ctx.close()


def _model(name, N=None, L=None):
    spec = synth.WORKLOADS[name]
    sh = spec["shape"]
    if N is not None:
        sh = synth.ModelShape(N=N, C=16, D=sh.D, H=sh.H, F=sh.F, L=L if L is not None else sh.L)
    counts = synth.group_counts(sh.N, spec["fractions"])
    w = synth.model_weights(sh, 9)
    layers = [tuple(bf(lw[k]) for k in ("w_qkv", "w_o", "w_1", "w_2")) for lw in w["layers"]]
    return spec, sh, counts, w, layers


def _run_sharded(G, spec, sh, counts, w, layers, regroup, fused=False):
    from token_sparse_denoising_layer_b200.shard import ShardRank, link_local, run_local

    ranks = [ShardRank(r, G, sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]),
                       spec["T"], spec["budgets"], counts, shift=spec["shift"]) for r in range(G)]
    if fused:
        link_local(ranks)
    x0 = synth.latent(sh.N, 16, 9)
    g0 = synth.random_split(sh.N, counts, 9)
    for rk in ranks:
        rk.reset(dev(x0), dev(g0))
    for i in range(spec["T"]):
        run_local([rk.steps(i, regroup) for rk in ranks])
    for rk in ranks:
        abi.hsa_sync_check(rk.ctx)
    out = [host(rk.x) for rk in ranks]
    g = [host(rk.g) for rk in ranks]
    for rk in ranks:
        rk.close()
    return x0, g0, out, g


def _run_single(spec, sh, counts, w, layers, x0, g0, regroup):
    from token_sparse_denoising_layer_b200.loop import HsaLoop

    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]), spec["T"],
                   spec["budgets"], counts, shift=spec["shift"])
    loop.reset(x0, g0)
    loop.run(regroup=regroup)
    abi.hsa_sync_check(loop.ctx)
    x = host(loop.x)
    loop.close()
    return x


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("G", [1, 2, 3])
@pytest.mark.parametrize("regroup", [False, True])
def test_sharded_tiny_dit_matches_single_gpu_loop(G, regroup):
    need_gpu()
    spec, sh, counts, w, layers = _model("tiny_dit")
    x0, g0, xs, gs = _run_sharded(G, spec, sh, counts, w, layers, regroup)
    for r in range(1, G):
        assert np.array_equal(xs[r], xs[0]) and np.array_equal(gs[r], gs[0])
    x1 = _run_single(spec, sh, counts, w, layers, x0, g0, regroup)
    d = _rel(xs[0], x1)
    print(f"G={G} regroup={regroup}: sharded vs single-GPU loop {d:.2e} "
          f"(bitwise: {np.array_equal(xs[0], x1)})")
    assert d <= 1e-2
    xr = O.run_loop(w, x0, g0, spec["T"], list(spec["budgets"]), counts,
                    O.sigma_schedule(spec["T"], spec["shift"]), sh.H, regroup=regroup)
    assert _rel(xs[0], xr) <= 2e-2


def test_sharded_dit30_shapes_three_ranks():
    """The 30-layer DiT's D, H, F, T and budgets with one layer and N = 840:
    several 128-row tiles per rank and ragged chunks (a = 840, 588, 336)."""
    need_gpu()
    spec, sh, counts, w, layers = _model("dit30_1536", N=840, L=1)
    x0, g0, xs, gs = _run_sharded(3, spec, sh, counts, w, layers, True)
    assert np.array_equal(xs[1], xs[0]) and np.array_equal(xs[2], xs[0])
    x1 = _run_single(spec, sh, counts, w, layers, x0, g0, True)
    d = _rel(xs[0], x1)
    print(f"dit30 shapes, G=3: sharded vs single-GPU loop {d:.2e}")
    assert d <= 1e-2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_sharded_world_of_one_through_nccl():
    """run_dist over a real NCCL process group of size 1 equals the in-process
    driver bit for bit."""
    need_gpu()
    import torch.distributed as dist

    from token_sparse_denoising_layer_b200.shard import ShardRank, run_dist

    spec, sh, counts, w, layers = _model("tiny_dit")
    x0, g0, xs, _ = _run_sharded(1, spec, sh, counts, w, layers, True)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True,
                          timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        rk = ShardRank(0, 1, sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]),
                       spec["T"], spec["budgets"], counts, shift=spec["shift"])
        rk.reset(dev(x0), dev(g0))
        for i in range(spec["T"]):
            run_dist(rk.steps(i, True))
        abi.hsa_sync_check(rk.ctx)
        assert np.array_equal(host(rk.x), xs[0])
        rk.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("G,fused", [(1, False), (2, False), (3, False), (2, True), (3, True)])
def test_sharded_conditioned_step(G, fused):
    """Conditioned blocks (per-iteration modulation of every layer, text
    cross-attention in every layer) in the sharded step: every rank ends with
    the same latent bit for bit, equal to the single-GPU conditioned loop
    (hsa_step_cond) within rounding, and to the float64 oracle within 2e-2."""
    need_gpu()
    from token_sparse_denoising_layer_b200.loop import HsaLoop
    from token_sparse_denoising_layer_b200.shard import ShardRank, link_local, run_local

    spec, sh, counts, w, layers = _model("tiny_dit")
    T, L = spec["T"], sh.L
    mods = [[synth.modulation(sh.D, 300 + i * L + l, spread=0.3) for l in range(L)]
            for i in range(T)]
    cross = [synth.cross_attention_weights(sh.D, 16, 400 + l) for l in range(L)]
    mods_dev = [[dev(m) for m in row] for row in mods]
    xa = [abi.cross_attn(bf(c["w_q"]), bf(c["w_o"]), bf(c["k_txt"]), bf(c["v_txt"]), 16)
          for c in cross]
    conds = [abi.StepCond(mods_dev[i], xa) for i in range(T)]
    x0 = synth.latent(sh.N, 16, 9)
    g0 = synth.random_split(sh.N, counts, 9)
    ranks = [ShardRank(r, G, sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]),
                       T, spec["budgets"], counts, shift=spec["shift"]) for r in range(G)]
    if fused:
        link_local(ranks)
    for rk in ranks:
        rk.reset(dev(x0), dev(g0))
    for i in range(T):
        run_local([rk.steps(i, True, cond=conds[i]) for rk in ranks])
    for rk in ranks:
        abi.hsa_sync_check(rk.ctx)
    xs = [host(rk.x) for rk in ranks]
    for rk in ranks:
        rk.close()
    for r in range(1, G):
        assert np.array_equal(xs[r], xs[0])
    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]), T,
                   spec["budgets"], counts, shift=spec["shift"])
    loop.reset(x0, g0)
    for i in range(T):
        loop.step(i, True, cond=conds[i])
    abi.hsa_sync_check(loop.ctx)
    x1 = host(loop.x)
    loop.close()
    d = _rel(xs[0], x1)
    print(f"conditioned, G={G}: sharded vs single-GPU loop {d:.2e} "
          f"(bitwise: {np.array_equal(xs[0], x1)})")
    assert d <= 1e-2
    xr = O.run_loop(w, x0, g0, T, list(spec["budgets"]), counts,
                    O.sigma_schedule(T, spec["shift"]), sh.H, mods=mods, cross=cross)
    assert _rel(xs[0], xr) <= 2e-2


# --------------------------------------------------------------------------- fused K|V exchange


@pytest.mark.parametrize("N,D,a", [(700, 256, 333), (8192, 1536, 4097), (8192, 1536, 129)])
@pytest.mark.parametrize("G", [1, 3, 8])
def test_qkv_project_peers_writes_every_copy(N, D, a, G):
    """hsa_qkv_project_peers: the same Q as hsa_qkv_project, bit for bit, and in
    every one of the G cache pairs the same fresh rows at A and the copy's own
    stale rows elsewhere; the rows also match the float64 oracle."""
    need_gpu()
    H = D // 128
    ctx = abi.hsa_create(N=N, D=D, H=H, F=4 * D, L=1, T=1, budgets=[1], counts=[N])
    w = synth.layer_weights(D, 64, 5)
    x = synth.hidden_rows(N, D, 5)
    idx = synth.random_active_set(N, a, 5)
    u = torch.empty((a, D), dtype=torch.bfloat16, device="cuda")
    abi.hsa_ln_gather(ctx, dev(x), dev(idx), a, u)
    wq = bf(w["w_qkv"])
    ks, vs = synth.stale_kv(N, D, 5)
    q1 = torch.empty((a, D), dtype=torch.bfloat16, device="cuda")
    kc1, vc1 = bf(ks), bf(vs)
    abi.hsa_qkv_project(ctx, wq, u, dev(idx), a, q1, kc1, vc1)
    stale = [synth.stale_kv(N, D, 50 + g) for g in range(G)]
    kcs = [bf(k) for k, _ in stale]
    vcs = [bf(v) for _, v in stale]
    q = torch.empty((a, D), dtype=torch.bfloat16, device="cuda")
    abi.hsa_qkv_project_peers(ctx, wq, u, dev(idx), a, q, kcs, vcs)
    abi.hsa_sync_check(ctx)
    assert torch.equal(q, q1)
    rest = np.setdiff1d(np.arange(N), idx)
    k1, v1 = host(kc1), host(vc1)
    for g in range(G):
        kg, vg = host(kcs[g]), host(vcs[g])
        assert (kg[idx] == k1[idx]).all() and (vg[idx] == v1[idx]).all()
        assert (kg[rest] == stale[g][0][rest]).all() and (vg[rest] == stale[g][1][rest]).all()
    qkv = O.linear(O.layer_norm(x[idx]), w["w_qkv"])
    assert normwise(host(q), qkv[:, :D]) <= BF16_TOL
    assert normwise(k1[idx], qkv[:, D:2 * D]) <= BF16_TOL
    assert normwise(v1[idx], qkv[:, 2 * D:]) <= BF16_TOL
    ctx.close()


def test_qkv_project_peers_rejects_bad_cache_lists():
    need_gpu()
    N, D = 256, 128
    ctx = abi.hsa_create(N=N, D=D, H=1, F=512, L=1, T=1, budgets=[1], counts=[N])
    u = torch.zeros((8, D), dtype=torch.bfloat16, device="cuda")
    q = torch.empty_like(u)
    wq = torch.zeros((3 * D, D), dtype=torch.bfloat16, device="cuda")
    idx = torch.arange(8, dtype=torch.int32, device="cuda")
    kc = torch.zeros((N, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    for ks, vs in (([], []), ([kc] * 9, [vc] * 9), ([kc, kc.data_ptr() + 2], [vc, vc]),
                   ([kc, 0], [vc, vc])):
        with pytest.raises(abi.HsaError) as e:
            abi.hsa_qkv_project_peers(ctx, wq, u, idx, 8, q, ks, vs)
        assert e.value.status == 1
    abi.hsa_sync_check(ctx)
    ctx.close()


def test_qkv_project_peers_skips_and_reports_bad_rows():
    """Indices outside [0, N) are skipped in every copy and reported by
    hsa_sync_check; the valid rows and Q are written as by hsa_qkv_project."""
    need_gpu()
    N, D, G = 256, 128, 3
    ctx = abi.hsa_create(N=N, D=D, H=1, F=512, L=1, T=1, budgets=[1], counts=[N])
    w = synth.layer_weights(D, 64, 7)
    idx = np.array([1, 2, -1, 300, 5, 255], dtype=np.int32)
    n = len(idx)
    u = bf(synth.bf16_round(synth.rng(7).standard_normal((n, D), dtype=np.float32)))
    wq = bf(w["w_qkv"])
    ks, vs = synth.stale_kv(N, D, 7)
    q1 = torch.empty((n, D), dtype=torch.bfloat16, device="cuda")
    kc1, vc1 = bf(ks), bf(vs)
    abi.hsa_qkv_project(ctx, wq, u, dev(idx), n, q1, kc1, vc1)
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_sync_check(ctx)
    assert e.value.status == 7
    kcs = [bf(ks) for _ in range(G)]
    vcs = [bf(vs) for _ in range(G)]
    q = torch.empty((n, D), dtype=torch.bfloat16, device="cuda")
    abi.hsa_qkv_project_peers(ctx, wq, u, dev(idx), n, q, kcs, vcs)
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_sync_check(ctx)
    assert e.value.status == 7
    assert torch.equal(q, q1)
    good = np.array([1, 2, 5, 255])
    rest = np.setdiff1d(np.arange(N), good)
    for g in range(G):
        assert torch.equal(kcs[g], kc1) and torch.equal(vcs[g], vc1)
        assert (host(kcs[g])[rest] == ks[rest]).all()
    assert not (host(kc1)[good] == ks[good]).all()
    ctx.close()


@pytest.mark.parametrize("G", [1, 2, 3])
@pytest.mark.parametrize("regroup", [False, True])
def test_sharded_fused_exchange_matches_all_gather(G, regroup):
    """Ranks whose QKV epilogue writes every rank's cache end bit for bit where
    the all-gather path ends, on every rank."""
    need_gpu()
    spec, sh, counts, w, layers = _model("tiny_dit")
    _, _, xg, gg = _run_sharded(G, spec, sh, counts, w, layers, regroup)
    _, _, xf, gf = _run_sharded(G, spec, sh, counts, w, layers, regroup, fused=True)
    for r in range(G):
        assert np.array_equal(xf[r], xg[0]) and np.array_equal(gf[r], gg[0])


def test_sharded_fused_dit30_shapes_three_ranks():
    need_gpu()
    spec, sh, counts, w, layers = _model("dit30_1536", N=840, L=2)
    _, _, xg, _ = _run_sharded(3, spec, sh, counts, w, layers, True)
    _, _, xf, _ = _run_sharded(3, spec, sh, counts, w, layers, True, fused=True)
    for r in range(3):
        assert np.array_equal(xf[r], xg[0])


def test_sharded_fused_world_of_one_through_nccl():
    """The fused exchange across processes (caches linked by CUDA IPC, the
    barrier a one-element NCCL all-reduce) in a world of one equals the
    in-process driver bit for bit."""
    need_gpu()
    import torch.distributed as dist

    from token_sparse_denoising_layer_b200.shard import ShardRank, link_ipc, run_dist

    spec, sh, counts, w, layers = _model("tiny_dit")
    x0, g0, xs, _ = _run_sharded(1, spec, sh, counts, w, layers, True)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True,
                          timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        rk = ShardRank(0, 1, sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]),
                       spec["T"], spec["budgets"], counts, shift=spec["shift"])
        link_ipc(rk)
        rk.reset(dev(x0), dev(g0))
        for i in range(spec["T"]):
            run_dist(rk.steps(i, True))
        abi.hsa_sync_check(rk.ctx)
        assert np.array_equal(host(rk.x), xs[0])
        rk.close()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()


def _ipc_writer_rank(rank, port, out):
    """One of two processes on GPU 0: both link their caches through CUDA IPC;
    rank 1 runs the multi-copy QKV store into its own cache and rank 0's; rank
    0 then checks its cache against a single-copy projection of its own."""
    import gc
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import datetime as dt

    import torch as th
    import torch.distributed as dist

    from token_sparse_denoising_layer_b200 import abi as A
    from token_sparse_denoising_layer_b200 import synth as S
    from token_sparse_denoising_layer_b200.shard import open_peer_caches

    ok, msg = False, ""
    try:
        th.cuda.set_device(0)
        store = dist.TCPStore("127.0.0.1", port, 2, rank == 0, timeout=dt.timedelta(seconds=60))
        dist.init_process_group("gloo", store=store, rank=rank, world_size=2,
                                timeout=dt.timedelta(seconds=60))
        N, D, a = 700, 256, 333
        ctx = A.hsa_create(N=N, D=D, H=2, F=512, L=1, T=1, budgets=[1], counts=[N])
        bf16 = lambda x: th.from_numpy(x).cuda().to(th.bfloat16)
        ks0, vs0 = S.stale_kv(N, D, 60 + rank)
        kc, vc = bf16(ks0), bf16(vs0)
        kl, vl, keep = open_peer_caches([kc], [vc])
        w = S.layer_weights(D, 64, 8)
        idx = th.from_numpy(S.random_active_set(N, a, 8)).cuda()
        u = bf16(S.bf16_round(S.rng(8).standard_normal((a, D), dtype=np.float32)))
        wq = bf16(w["w_qkv"])
        q = th.empty((a, D), dtype=th.bfloat16, device="cuda")
        th.cuda.synchronize()
        dist.barrier()
        if rank == 1:
            A.hsa_qkv_project_peers(ctx, wq, u, idx, a, q, kl[0], vl[0])
            A.hsa_sync_check(ctx)
            th.cuda.synchronize()
        dist.barrier()  # rank 1's stores into rank 0's cache are complete
        if rank == 0:
            kr, vr = bf16(ks0), bf16(vs0)
            A.hsa_qkv_project(ctx, wq, u, idx, a, q, kr, vr)
            A.hsa_sync_check(ctx)
            ok = bool(th.equal(kc, kr) and th.equal(vc, vr))
            rest = np.setdiff1d(np.arange(N), idx.cpu().numpy())
            ok = ok and bool((kc.float().cpu().numpy()[rest] == ks0[rest]).all())
            msg = "rank 0 cache equals the single-copy projection" if ok else "mismatch"
        else:
            ok, msg = True, "writer"
        dist.barrier()  # rank 0 has read its cache before the mappings go
        del keep, kl, vl
        gc.collect()
        th.cuda.synchronize()
        dist.barrier()  # both mappings released before either cache is freed
        th.cuda.ipc_collect()
        dist.barrier()
        ctx.close()
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        msg = repr(e)
    out.put((rank, ok, msg))


def test_ipc_peer_stores_between_two_processes():
    """The multi-copy QKV store through a CUDA IPC mapping of another process's
    cache: two processes on one GPU, synchronised on the host only (no kernel
    waits on the other process)."""
    need_gpu()
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_writer_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(2))
    for p in procs:
        p.join(60)
    print(res)
    assert all(p.exitcode == 0 for p in procs)
    assert [r for r, _, _ in res] == [0, 1]
    assert all(ok for _, ok, _ in res), res
