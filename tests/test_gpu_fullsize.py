"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (hsa_layer_forward / hsa_step), checked on sampled outputs the oracle
computes one by one (tests/sampled_block.py, itself checked against the
oracle's whole block on small cases).

Where the oracle can afford it, it builds the exact KV cache the sampled
queries see: every active row's fresh K and V (float64), stale rows elsewhere.
For the 40-layer DiT's layer at 25% and 100% active (18900 and 75600 of 75600
rows at D = 5120) it checks the GPU's fresh K/V rows on a sample first, then
attends against the cache as the GPU wrote it.  Skipped rows of x and of the
caches must be untouched, bit for bit.
"""

import numpy as np
import pytest

from gpu_util import BF16_TOL, bf, dev, host, need_gpu, normwise, torch
import sampled_block as SB
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import abi, synth

pytestmark = pytest.mark.gpu


def _device_weights(D, F, seed):
    w = synth.layer_weights(D, F, seed)
    return w, abi.layer_weights(*(bf(w[k]) for k in ("w_qkv", "w_o", "w_1", "w_2")))


@pytest.mark.parametrize("name,N,D,H,F,a,n_sample,via_gpu_cache", [
    ("layer_1536 f=1", 32760, 1536, 12, 6144, 32760, 192, False),
    ("layer_1536 f=0.5", 32760, 1536, 12, 6144, 16380, 128, False),
    ("layer_1536 f=0.25", 32760, 1536, 12, 6144, 8190, 128, False),
    ("layer_1536 f=0.1", 32760, 1536, 12, 6144, 3276, 192, False),
    ("dit30 layer, 40% active", 32760, 1536, 12, 8960, 13104, 128, False),
    ("dit40 layer, 2048 active", 75600, 5120, 40, 13824, 2048, 48, False),
    ("dit40 layer, 25% active", 75600, 5120, 40, 13824, 18900, 64, True),
    ("dit40 layer, 100% active", 75600, 5120, 40, 13824, 75600, 64, True),
])
def test_layer_full_size_sampled(name, N, D, H, F, a, n_sample, via_gpu_cache):
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
    xg = host(xd)
    n_rows = idx[rows]
    if via_gpu_cache:
        # the fresh K/V rows on a wider sample first, then attention against
        # the cache the GPU wrote (the sampled rows of which are now checked)
        kv_rows = np.unique(np.r_[rows, np.sort(r.choice(a, size=min(512, a), replace=False))])
        k_ref, v_ref = SB.kv_rows(w, x, idx, kv_rows)
        kg, vg = host(kc), host(vc)
        assert normwise(kg[idx[kv_rows]], k_ref) <= BF16_TOL, name
        assert normwise(vg[idx[kv_rows]], v_ref) <= BF16_TOL, name
        x_ref = SB.block_rows_given_cache(w, x, idx, kg, vg, H, rows)
        del kg, vg
    else:
        x_ref, k_ref, v_ref = SB.block_rows(w, x, idx, ks, vs, H, rows)
        assert normwise(host(kc)[n_rows], k_ref) <= BF16_TOL
        assert normwise(host(vc)[n_rows], v_ref) <= BF16_TOL
    err = normwise(xg[n_rows] - x[n_rows], x_ref - x[n_rows])
    print(f"{name}: block output error {err:.2e} on {len(rows)} sampled rows")
    assert err <= BF16_TOL, name
    skipped = np.setdiff1d(np.arange(N), idx)
    if len(skipped):
        s = r.choice(skipped, size=min(512, len(skipped)), replace=False)
        assert (xg[s] == x[s]).all()
        assert (host(kc)[s] == ks[s]).all() and (host(vc)[s] == vs[s]).all()
    ctx.close()


@pytest.mark.parametrize("workload,seed,regroup", [
    ("dit30_1536", 3, False), ("dit30_1536", 3, True), ("dit40_5120", 4, True)])
def test_reduced_shape_loop(workload, seed, regroup):
    """The whole loop at a large workload's D, H, F, T, shift and budgets (the
    30-layer DiT: 1536 wide, {40, 20, 10} at 40/30/30; the 40-layer DiT: 5120
    wide, {40, 10} at 25/75), with L = 2 layers and a 21x8x10 latent
    (N = 1680).  Every iteration is checked
    (loop_check.run_checked: schedule of the GPU's groups; bit-exact scores
    and assignment at every re-grouping); x_T is compared with the float64 oracle's loop."""
    need_gpu()
    from loop_check import run_checked
    from token_sparse_denoising_layer_b200.loop import HsaLoop

    spec = synth.WORKLOADS[workload]
    big = spec["shape"]
    sh = synth.ModelShape(N=1680, C=16, D=big.D, H=big.H, F=big.F, L=2)
    T, budgets = spec["T"], list(spec["budgets"])
    counts = synth.group_counts(sh.N, spec["fractions"])
    w = synth.model_weights(sh, seed)
    layers = [tuple(bf(lw[k]) for k in ("w_qkv", "w_o", "w_1", "w_2")) for lw in w["layers"]]
    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]), T, budgets,
                   counts, shift=spec["shift"])
    x0 = synth.latent(sh.N, 16, seed)
    g0 = synth.random_split(sh.N, counts, seed)
    loop.reset(x0, g0)
    n_regroup, moved = run_checked(loop, T, budgets, counts, g0, regroup=regroup)
    log = []
    xr = O.run_loop(w, x0, g0, T, budgets, counts, O.sigma_schedule(T, spec["shift"]), sh.H,
                    regroup=regroup, log=log)
    drift = float(np.linalg.norm(host(loop.x) - xr) / np.linalg.norm(xr))
    parted = int((host(loop.g) != log[-1]["g"]).sum())
    print(f"{workload} shapes (L=2, N=1680, T={T}, regroup={regroup}): x_T drift vs float64 "
          f"oracle {drift:.3e}; {n_regroup} re-groupings moved {moved} group ids; final "
          f"groups differ from the oracle's on {parted} of {sh.N} tokens")
    assert drift <= 2e-2
    loop.close()
