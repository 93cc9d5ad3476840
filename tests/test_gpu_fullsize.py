"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (hsa_layer_forward / hsa_step), checked on sampled outputs the oracle
computes one by one.

The oracle builds the exact KV cache the sampled queries see: every active
row's fresh K and V (float64), stale rows elsewhere.  Then, for sampled active
rows, it runs attention against that cache and the rest of the block.
Skipped rows of x and of the caches must be untouched, bit for bit.
"""

import numpy as np
import pytest

from gpu_util import BF16_TOL, bf, dev, host, need_gpu, normwise, torch
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import abi, synth

pytestmark = pytest.mark.gpu


def _device_weights(D, F, seed):
    w = synth.layer_weights(D, F, seed)
    return w, abi.layer_weights(*(bf(w[k]) for k in ("w_qkv", "w_o", "w_1", "w_2")))


def _sampled_block_reference(w, x, idx, ks, vs, H, rows):
    """Oracle block outputs for the active rows idx[rows], given the full cache update."""
    D = x.shape[1]
    u = O.layer_norm(x[idx])                               # all active rows: K, V into the cache
    kv = O.linear(u, w["w_qkv"][D:])
    kc = ks.astype(np.float64)
    vc = vs.astype(np.float64)
    kc[idx] = kv[:, :D]
    vc[idx] = kv[:, D:]
    q = O.linear(u[rows], w["w_qkv"][:D])
    o = O.attention(q, kc, vc, H)
    x1 = x[idx[rows]].astype(np.float64) + O.linear(o, w["w_o"])
    x2 = x1 + O.linear(O.gelu(O.linear(O.layer_norm(x1), w["w_1"])), w["w_2"])
    return x2, kc[idx[rows]], vc[idx[rows]]


@pytest.mark.parametrize("name,N,D,H,F,a,n_sample", [
    ("layer_1536 f=1", 32760, 1536, 12, 6144, 32760, 192),
    ("layer_1536 f=0.1", 32760, 1536, 12, 6144, 3276, 192),
    ("dit30 layer, 40% active", 32760, 1536, 12, 8960, 13104, 128),
    ("dit40 layer, 2048 active", 75600, 5120, 40, 13824, 2048, 48),
])
def test_layer_full_size_sampled(name, N, D, H, F, a, n_sample):
    need_gpu()
    ctx = abi.hsa_create(N=N, D=D, H=H, F=F, L=1, T=1, budgets=[1], counts=[N])
    w, lw = _device_weights(D, F, 21)
    x = synth.hidden_rows(N, D, 21)
    ks, vs = synth.stale_kv(N, D, 21)
    idx = synth.random_active_set(N, a, 21)
    xd, kc, vc = dev(x), bf(ks), bf(vs)
    abi.hsa_layer_forward(ctx, lw, xd, dev(idx), a, kc, vc)
    abi.hsa_sync_check(ctx)
    r = synth.rng(5)
    rows = np.sort(r.choice(a, size=min(n_sample, a), replace=False))
    if a > 1 and 0 not in rows:
        rows[0] = 0                       # the first and the last active row
    if a - 1 not in rows:
        rows[-1] = a - 1
    rows = np.unique(rows)
    x_ref, k_ref, v_ref = _sampled_block_reference(w, x, idx, ks, vs, H, rows)
    xg = host(xd)
    n_rows = idx[rows]
    assert normwise(xg[n_rows] - x[n_rows], x_ref - x[n_rows]) <= BF16_TOL, name
    assert normwise(host(kc)[n_rows], k_ref) <= BF16_TOL
    assert normwise(host(vc)[n_rows], v_ref) <= BF16_TOL
    skipped = np.setdiff1d(np.arange(N), idx)
    if len(skipped):
        s = r.choice(skipped, size=min(512, len(skipped)), replace=False)
        assert (xg[s] == x[s]).all()
        assert (host(kc)[s] == ks[s]).all() and (host(vc)[s] == vs[s]).all()
    ctx.close()


def test_dit30_shapes_loop_drift():
    """The whole loop at the 30-layer DiT's D, H, F, T, shift and budgets, with
    one layer and a 21x5x8 latent (N = 840), against the float64 oracle."""
    need_gpu()
    spec = synth.WORKLOADS["dit30_1536"]
    sh = synth.ModelShape(N=840, C=16, D=1536, H=12, F=8960, L=1)
    T, budgets = spec["T"], list(spec["budgets"])
    counts = synth.group_counts(sh.N, spec["fractions"])
    w = synth.model_weights(sh, 3)
    layers = [tuple(bf(lw[k]) for k in ("w_qkv", "w_o", "w_1", "w_2")) for lw in w["layers"]]
    from token_sparse_denoising_layer_b200.loop import HsaLoop
    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]), T, budgets,
                   counts, shift=spec["shift"])
    x0 = synth.latent(sh.N, 16, 3)
    g0 = synth.random_split(sh.N, counts, 3)
    loop.reset(x0, g0)
    loop.run(regroup=False)
    abi.hsa_sync_check(loop.ctx)
    xr = O.run_loop(w, x0, g0, T, budgets, counts, O.sigma_schedule(T, spec["shift"]), sh.H,
                    regroup=False)
    drift = float(np.linalg.norm(host(loop.x) - xr) / np.linalg.norm(xr))
    print(f"dit30-shape loop (L=1, N=840, T=40) x_T drift vs float64 oracle: {drift:.3e}")
    assert drift <= 2e-2
    loop.close()


def test_dit40_shapes_loop_drift():
    """The whole loop at the 40-layer DiT's D, H, F, T, shift and budgets ({40, 10}
    at 25/75%), with one layer and N = 210 tokens, against the float64 oracle."""
    need_gpu()
    spec = synth.WORKLOADS["dit40_5120"]
    sh = synth.ModelShape(N=210, C=16, D=5120, H=40, F=13824, L=1)
    T, budgets = spec["T"], list(spec["budgets"])
    counts = synth.group_counts(sh.N, spec["fractions"])
    w = synth.model_weights(sh, 4)
    layers = [tuple(bf(lw[k]) for k in ("w_qkv", "w_o", "w_1", "w_2")) for lw in w["layers"]]
    from token_sparse_denoising_layer_b200.loop import HsaLoop
    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]), T, budgets,
                   counts, shift=spec["shift"])
    x0 = synth.latent(sh.N, 16, 4)
    g0 = synth.random_split(sh.N, counts, 4)
    loop.reset(x0, g0)
    loop.run(regroup=False)
    abi.hsa_sync_check(loop.ctx)
    xr = O.run_loop(w, x0, g0, T, budgets, counts, O.sigma_schedule(T, spec["shift"]), sh.H,
                    regroup=False)
    drift = float(np.linalg.norm(host(loop.x) - xr) / np.linalg.norm(xr))
    print(f"dit40-shape loop (L=1, N=210, T=40) x_T drift vs float64 oracle: {drift:.3e}")
    assert drift <= 2e-2
    loop.close()
