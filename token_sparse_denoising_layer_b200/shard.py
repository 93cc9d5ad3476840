"""Sequence-sharded HSA step: one loop split over G ranks (one GPU each).

"Technical Summary: Heterogeneous Step Allocation (HSA) for Efficient Video
Generation", section 2.2: every active token writes fresh K/V rows into the
per-layer cache, then every active query attends to all N cached rows.  So
the active list A_i of a step splits across ranks with one exchange per
layer: each rank runs QKV, attention, out-projection and MLP for its share of
A_i, and the fresh K/V rows of all shares are gathered into every rank's copy
of the cache before attention reads it.

Partition.  A_i (ascending, identical on every rank because the group ids
are) is cut into G chunks of c positions, c = ceil(a / G) rounded up to a
multiple of 4 so that every chunk of the int32 list starts on a 16-byte
boundary; rank r takes positions [r c, min(a, (r+1) c)).  Only trailing
chunks can be short, so after an all-gather of c-row chunks the first a rows,
in rank order, are the fresh rows of A_i in order and scatter straight into
the cache by A_i.

Per step on rank r:
  schedule (all of A_i) -> embed, L x [LN, Q and K|V GEMMs of its chunk,
  all-gather K|V, scatter into the cache, attention of its queries against
  all N rows, out-projection, (text cross-attention), MLP; with the
  iteration's modulation when conditioned] -> head of its chunk into a zeroed [N, C]
  buffer -> all-reduce (sum) of that buffer, which is exact because every
  active row has exactly one non-zero contributor -> cached Euler over all N
  (replicated) -> re-grouping (replicated; deterministic, so the group ids
  stay identical on every rank).

Fused K|V exchange (``link_local`` / ``link_ipc``).  Instead of the
Q and K|V GEMMs, the all-gather and the scatter, one QKV GEMM per layer
(hsa_qkv_project_peers) stores every fresh K/V row of the rank's chunk
straight into row A_i[m] of every rank's copy of the cache: its own through
this GPU's memory, the others' through peer-mapped pointers over NVLink
(stores only; nothing loads another GPU's memory).  A device-side barrier
after it (a one-element all-reduce on the stream) keeps every rank's
attention from reading its cache before all ranks' writes are complete.  The
writes of step i + 1 cannot overtake a peer still reading step i's rows:
they start after the velocity all-reduce of step i, which completes only
once every rank has reached it, i.e. after all of that rank's step-i
attention.  Across processes the peers' caches are reached through CUDA IPC
mappings (point to point; no multicast object is created).

Every step of the path runs in libhsa's kernels; the exchanges are
collectives.  The step is written once, as a generator that yields each
exchange; `run_dist` serves the requests with torch.distributed (NCCL on
GPUs, gloo in CPU tests) and `run_local` serves G ranks held in one process
by copying between their buffers.
"""

from __future__ import annotations

from typing import Iterator, List, Sequence, Tuple

from . import abi
from .loop import sigma_schedule


CHUNK_ALIGN = 4  # int32 entries per 16 bytes


def chunk_rows(a: int, G: int) -> int:
    """Rows per rank for a active tokens: ceil(a / G), rounded up to CHUNK_ALIGN."""
    c = -(-a // G)
    return max(CHUNK_ALIGN, -(-c // CHUNK_ALIGN) * CHUNK_ALIGN)


def shard_slices(a: int, G: int) -> Tuple[int, List[Tuple[int, int]]]:
    """Chunk size c and each rank's (start, count) within the active list."""
    if G < 1 or a < 0:
        raise ValueError("need G >= 1 and a >= 0")
    c = chunk_rows(a, G)
    out = []
    for r in range(G):
        s = min(a, r * c)
        out.append((s, min(a, s + c) - s))
    return c, out


Request = Tuple  # ("all_gather", send, recv) | ("all_reduce_sum", buf) | ("barrier", buf)


class ShardRank:
    """One rank's device state for the sharded loop.

    The latent, velocity caches, group ids and the per-layer K/V caches are
    replicated ([N, ...] on every rank); the hidden rows h are [N, D] but a
    rank only touches the rows of its chunk.  ``layers`` holds the bf16 CUDA
    tensors (w_qkv, w_o, w_1, w_2) per block; w_in [D, C] and w_head [C, D]
    are float32.
    """

    def __init__(self, rank: int, G: int, N: int, D: int, H: int, F: int, layers, w_in, w_head,
                 T: int, budgets: Sequence[int], counts: Sequence[int], shift: float = 1.0,
                 m: int = 0, stream=None):
        import torch

        if not 0 <= rank < G:
            raise ValueError("rank outside [0, G)")
        self.torch = torch
        self.rank, self.G = rank, G
        self.N, self.D, self.H, self.F, self.L = N, D, H, F, len(layers)
        self.T, self.budgets, self.counts = T, list(budgets), list(counts)
        self.ctx = abi.hsa_create(N=N, D=D, H=H, F=F, L=self.L, T=T, budgets=budgets,
                                  counts=counts, m=m, stream=stream)
        f32 = dict(dtype=torch.float32, device="cuda")
        bf = dict(dtype=torch.bfloat16, device="cuda")
        self.x = torch.zeros((N, 16), **f32)
        self.v_hat = torch.zeros((N, 16), **f32)
        self.v_hat_prev = torch.zeros((N, 16), **f32)
        self.v_stage = torch.zeros((N, 16), **f32)
        self.score = torch.zeros((N,), **f32)
        self.g = torch.zeros((N,), dtype=torch.uint8, device="cuda")
        self.mask = torch.zeros((N,), dtype=torch.uint8, device="cuda")
        self.active_idx = torch.zeros((N,), dtype=torch.int32, device="cuda")
        self.h = torch.zeros((N, D), **f32)
        self.k_cache = [torch.zeros((N, D), **bf) for _ in layers]
        self.v_cache = [torch.zeros((N, D), **bf) for _ in layers]
        cmax = chunk_rows(N, G)
        self.u = torch.empty((cmax, D), **bf)
        self.q = torch.empty((cmax, D), **bf)
        self.o = torch.empty((cmax, D), **bf)
        self.kv_send = torch.empty((cmax, 2 * D), **bf)
        self.kv_recv = torch.empty((G * cmax, 2 * D), **bf)
        # fused exchange: layer l's cache of every rank, rank order (None: all-gather)
        self.peer_k = None
        self.peer_v = None
        self.sync = torch.zeros((1,), dtype=torch.int32, device="cuda")
        self._peers = None
        # W_qkv rows [0, D) project Q, rows [D, 3D) project K|V: contiguous views
        self.w_q = [lw[0][:D] for lw in layers]
        self.w_kv = [lw[0][D:] for lw in layers]
        self.layers = layers
        self.w_in, self.w_head = w_in, w_head
        self.sigmas = sigma_schedule(T, shift)

    def link_peer_caches(self, k_caches, v_caches) -> None:
        """Use the fused K|V exchange: ``k_caches[l]`` / ``v_caches[l]`` list
        layer l's cache of every rank in rank order (tensors or device
        addresses; this rank's entry is its own cache)."""
        if len(k_caches) != self.L or len(v_caches) != self.L:
            raise ValueError("need one list of caches per layer")
        for l in range(self.L):
            if len(k_caches[l]) != self.G or len(v_caches[l]) != self.G:
                raise ValueError("need one cache per rank in every layer")
            own = (abi._addr(k_caches[l][self.rank]), abi._addr(v_caches[l][self.rank]))
            if own != (self.k_cache[l].data_ptr(), self.v_cache[l].data_ptr()):
                raise ValueError("this rank's entry must be its own cache")
        self.peer_k = [list(k) for k in k_caches]
        self.peer_v = [list(v) for v in v_caches]

    def reset(self, x0, g0) -> None:
        """Start a run from latent x0 [N, 16] and group ids g0 [N] (same on every rank)."""
        t = self.torch
        self.x.copy_(t.as_tensor(x0))
        self.g.copy_(t.as_tensor(g0))
        for buf in (self.v_hat, self.v_hat_prev, self.v_stage, self.score):
            buf.zero_()

    def steps(self, i: int, regroup: bool = True, cond=None) -> Iterator[Request]:
        """Global iteration i on this rank; yields at each exchange.

        ``cond`` (abi.StepCond, or None) conditions the blocks as hsa_step_cond
        does: layer l's modulation rows of this iteration and its text
        cross-attention, run on the rank's own active rows (the text keys and
        values are the same on every rank, so cross-attention needs no
        exchange)."""
        ctx, D = self.ctx, self.D
        mods, cross = cond._keep if cond is not None else (None, None)
        a = abi.hsa_schedule(ctx, i, self.g, self.mask, self.active_idx)
        c, sl = shard_slices(a, self.G)
        s0, nr = sl[self.rank]
        idx_r = self.active_idx[s0:s0 + nr]
        abi.hsa_embed(ctx, self.w_in, self.x, idx_r, nr, self.h)
        for l in range(self.L):
            _, w_o, w_1, w_2 = self.layers[l]
            m = None if mods is None else mods[l]   # rows shift_a, scale_a, gate_a, shift_m, ...
            row = (lambda r: None) if m is None else (lambda r, m=m: m[r])
            abi.hsa_ln_gather_mod(ctx, self.h, idx_r, nr, self.u, row(0), row(1))
            if self.peer_k is not None:
                abi.hsa_qkv_project_peers(ctx, self.layers[l][0], self.u, idx_r, nr, self.q,
                                          self.peer_k[l], self.peer_v[l])
                yield ("barrier", self.sync)
            else:
                abi.hsa_linear(ctx, self.u, nr, D, self.w_q[l], D, self.q)
                abi.hsa_linear(ctx, self.u, nr, D, self.w_kv[l], 2 * D, self.kv_send)
                yield ("all_gather", self.kv_send[:c], self.kv_recv[:self.G * c])
                abi.hsa_kv_scatter_packed(ctx, self.kv_recv, self.active_idx, a,
                                          self.k_cache[l], self.v_cache[l])
            abi.hsa_attention(ctx, self.q, nr, self.k_cache[l], self.v_cache[l], self.o)
            abi.hsa_out_proj_residual_gated(ctx, w_o, self.o, idx_r, nr, self.h, row(2))
            xa = None if cross is None else cross[l]
            if xa is not None:
                w_qc, w_oc, k_txt, v_txt = xa._keep
                abi.hsa_ln_gather(ctx, self.h, idx_r, nr, self.u)
                abi.hsa_linear(ctx, self.u, nr, D, w_qc, D, self.q)
                abi.hsa_attention_kv(ctx, self.q, nr, k_txt, v_txt, xa.n_txt, self.o)
                abi.hsa_out_proj_residual(ctx, w_oc, self.o, idx_r, nr, self.h)
            abi.hsa_mlp_residual_mod(ctx, w_1, w_2, self.h, idx_r, nr, row(3), row(4), row(5))
        self.v_stage.zero_()
        abi.hsa_head(ctx, self.w_head, self.h, idx_r, nr, self.v_stage)
        yield ("all_reduce_sum", self.v_stage)
        s0, s1 = float(self.sigmas[i]), float(self.sigmas[i + 1])
        if regroup and self.T // self.budgets[-1] <= i < self.T - 1:
            # the Euler pass also writes the re-grouping scores, as hsa_step does
            abi.hsa_euler_step_score(ctx, self.x, self.v_hat, self.v_hat_prev, self.v_stage,
                                     self.mask, s0, s1, self.score)
            abi.hsa_select_from_score(ctx, self.score, self.g)
        else:
            abi.hsa_euler_step(ctx, self.x, self.v_hat, self.v_hat_prev, self.v_stage,
                               self.mask, s0, s1)

    def n_active(self, i: int) -> int:
        return abi.hsa_n_active(self.ctx, i)

    def close(self) -> None:
        self.ctx.close()
        self.peer_k = self.peer_v = None
        self._peers = None


def link_local(ranks: Sequence[ShardRank]) -> None:
    """Fused K|V exchange for ranks held in one process on one device: every
    rank's QKV epilogue writes all ranks' caches directly."""
    ks = [[rk.k_cache[l] for rk in ranks] for l in range(ranks[0].L)]
    vs = [[rk.v_cache[l] for rk in ranks] for l in range(ranks[0].L)]
    for rk in ranks:
        rk.link_peer_caches(ks, vs)


def open_peer_caches(k_caches, v_caches, group=None):
    """Every rank's copies of the per-layer caches as addresses valid in this
    process (collective over ``group``): this rank's tensors as they are, the
    other ranks' opened from their CUDA IPC handles, which map the peer's
    memory point to point (no multicast object).  Returns (ks, vs, keep):
    ks[l][r] and vs[l][r] for layer l of rank r, and the opened tensors, which
    must outlive every launch that stores through their addresses."""
    import torch.distributed as dist
    from torch.multiprocessing.reductions import reduce_tensor

    rank, G = dist.get_rank(group), dist.get_world_size(group)
    L = len(k_caches)
    mine = [(reduce_tensor(k), reduce_tensor(v)) for k, v in zip(k_caches, v_caches)]
    everyone = [None] * G
    dist.all_gather_object(everyone, mine, group=group)
    ks = [[None] * G for _ in range(L)]
    vs = [[None] * G for _ in range(L)]
    keep = []
    for r in range(G):
        if len(everyone[r]) != L:
            raise ValueError("ranks hold different numbers of layers")
        for l in range(L):
            if r == rank:
                ks[l][r], vs[l][r] = k_caches[l], v_caches[l]
                continue
            (fk, ak), (fv, av) = everyone[r][l]
            tk, tv = fk(*ak), fv(*av)
            keep += [tk, tv]
            ks[l][r], vs[l][r] = tk.data_ptr(), tv.data_ptr()
    return ks, vs, keep


def link_ipc(rk: ShardRank, group=None) -> None:
    """Fused K|V exchange across processes: every rank's caches reached through
    CUDA IPC peer mappings (collective over ``group``; ranks on GPUs of one
    NVLink domain, one process each)."""
    import torch.distributed as dist

    group = group or dist.group.WORLD
    if dist.get_world_size(group) != rk.G or dist.get_rank(group) != rk.rank:
        raise ValueError("group does not match the rank's (rank, G)")
    ks, vs, keep = open_peer_caches(rk.k_cache, rk.v_cache, group)
    rk._peers = keep
    rk.link_peer_caches(ks, vs)


def _serve_dist(req: Request, group) -> None:
    import torch.distributed as dist

    if req[0] == "all_gather":
        _, send, recv = req
        if dist.get_backend(group) == "nccl":
            dist.all_gather_into_tensor(recv, send, group=group)
        else:
            dist.all_gather(list(recv.chunk(dist.get_world_size(group))), send, group=group)
    elif req[0] == "all_reduce_sum":
        dist.all_reduce(req[1], op=dist.ReduceOp.SUM, group=group)
    elif req[0] == "barrier":
        # stream-ordered: completes only after every rank's earlier kernels
        dist.all_reduce(req[1], op=dist.ReduceOp.SUM, group=group)
    else:
        raise ValueError(f"unknown exchange {req[0]!r}")


def run_dist(steps: Iterator[Request], group=None) -> None:
    """Drive one rank's step generator with torch.distributed collectives.

    Every rank yields the same requests in the same order (the same number of
    layers, one reduction per step), so the collectives match across ranks."""
    for req in steps:
        _serve_dist(req, group)


def run_local(all_steps: Sequence[Iterator[Request]]) -> None:
    """Drive G ranks held in one process in lockstep, exchanging by copies."""
    gens = list(all_steps)
    while True:
        reqs = []
        for g in gens:
            try:
                reqs.append(next(g))
            except StopIteration:
                reqs.append(None)
        if all(r is None for r in reqs):
            return
        if any(r is None for r in reqs) or len({r[0] for r in reqs}) != 1:
            raise RuntimeError("ranks diverged: different exchange requests")
        op = reqs[0][0]
        if op == "all_gather":
            for _, _, recv in reqs:
                for r, (_, send, _) in enumerate(reqs):
                    recv[r * send.shape[0]:(r + 1) * send.shape[0]].copy_(send)
        elif op == "barrier":
            pass  # one process, one stream: the writes are already ordered
        elif op == "all_reduce_sum":
            total = reqs[0][1].clone()
            for r in reqs[1:]:
                total += r[1]
            for r in reqs:
                r[1].copy_(total)
        else:
            raise ValueError(f"unknown exchange {op!r}")
