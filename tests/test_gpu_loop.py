"""The whole HSA loop on the GPU (hsa_step) against the oracle's loop, on the
tiny DiT workload (4x8x8 latent, N=256, 2 layers, T=8, budgets {8, 4}).

The GPU runs the layers in bf16 and the oracle in float64, so the latents
drift apart by rounding; the drift after T steps is stated and bounded here.
With re-grouping on, a rounding difference can move a token whose score sits
on a group boundary, so the two runs' groups may part; what is unique is
checked step by step instead: at every iteration the GPU's active list is the
oracle's schedule of the GPU's groups, and after every re-grouping the GPU's
score buffer is the oracle's float32 L1 relative change of the GPU's own two
cached velocities, bit for bit, and the GPU's groups are the oracle's
assignment of that buffer.
"""

import numpy as np
import pytest

from gpu_util import bf, dev, host, need_gpu, torch
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import abi, synth
from token_sparse_denoising_layer_b200.loop import HsaLoop, sigma_schedule
from loop_check import run_checked

pytestmark = pytest.mark.gpu


def _setup(budgets=(8, 4), fractions=(0.5, 0.5), m=0):
    spec = synth.WORKLOADS["tiny_dit"]
    sh = spec["shape"]
    T = spec["T"]
    counts = synth.group_counts(sh.N, fractions)
    w = synth.model_weights(sh, spec["seed"])
    layers = [tuple(bf(lw[k]) for k in ("w_qkv", "w_o", "w_1", "w_2")) for lw in w["layers"]]
    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]), T,
                   list(budgets), counts, shift=spec["shift"], m=m)
    x0 = synth.latent(sh.N, 16, spec["seed"])
    g0 = synth.random_split(sh.N, counts, spec["seed"])
    return sh, T, counts, w, loop, x0, g0


def _drift(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))



def test_sigma_tables_agree():
    for T, s in ((8, 1.0), (40, 5.0)):
        assert (sigma_schedule(T, s) == O.sigma_schedule(T, s)).all()


@pytest.mark.parametrize("regroup", [False, True])
def test_tiny_dit_loop_drift(regroup):
    need_gpu()
    sh, T, counts, w, loop, x0, g0 = _setup()
    loop.reset(x0, g0)
    loop.run(regroup=regroup)
    abi.hsa_sync_check(loop.ctx)
    xg = host(loop.x)
    g_end = host(loop.g)
    assert [int((g_end == k).sum()) for k in range(2)] == counts
    xr = O.run_loop(w, x0, g0, T, [8, 4], counts, O.sigma_schedule(T, 1.0), sh.H, regroup=regroup)
    d = _drift(xg, xr)
    print(f"tiny DiT x_T drift vs float64 oracle (regroup={regroup}): {d:.3e}")
    assert d <= (2e-2 if not regroup else 5e-2)


def test_tiny_dit_regrouping_exact_at_every_step():
    """Re-grouping on, the tiny DiT loop checked iteration by iteration (see
    ``run_checked``), then its x_T against the oracle's loop."""
    need_gpu()
    sh, T, counts, w, loop, x0, g0 = _setup()
    loop.reset(x0, g0)
    n_regroup, moved = run_checked(loop, T, [8, 4], counts, g0)
    assert n_regroup == T - 1 - O.regroup_from(T, [8, 4])
    assert moved > 0                      # the groups really do change
    xr = O.run_loop(w, x0, g0, T, [8, 4], counts, O.sigma_schedule(T, 1.0), sh.H)
    d = _drift(host(loop.x), xr)
    print(f"tiny DiT, re-grouping checked per step: {n_regroup} re-groupings moved "
          f"{moved} group ids; x_T drift {d:.3e}")
    assert d <= 2e-2


def test_all_active_loop_matches_dense_oracle():
    """Every s_k = T: the GPU loop is uniform flow matching; compared with the
    oracle's dense loop (no KV cache, no velocity cache)."""
    need_gpu()
    sh, T, counts, w, loop, x0, g0 = _setup(budgets=(8,), fractions=(1.0,))
    loop.reset(x0, np.zeros(sh.N, dtype=np.uint8))
    loop.run()
    xr = O.dense_loop(w, x0, T, O.sigma_schedule(T, 1.0), sh.H)
    d = _drift(host(loop.x), xr)
    print(f"all-active loop drift vs dense oracle: {d:.3e}")
    assert d <= 2e-2


def test_loop_is_deterministic():
    need_gpu()
    sh, T, counts, w, loop, x0, g0 = _setup()
    loop.reset(x0, g0)
    loop.run()
    a = host(loop.x).copy()
    loop.reset(x0, g0)
    for kc in loop.k_cache + loop.v_cache:
        kc.zero_()
    loop.run()
    assert (host(loop.x) == a).all()


def test_phase_window_loop_drift():
    """Phase-aware window (first and last m iterations run all tokens) through
    the whole loop, against the oracle with the same window."""
    need_gpu()
    sh, T, counts, w, loop, x0, g0 = _setup(budgets=(8, 4, 2), fractions=(0.4, 0.3, 0.3), m=2)
    assert [loop.n_active(i) for i in range(T)] == [
        O.n_active(i, T, [8, 4, 2], counts, 2) for i in range(T)]
    assert loop.n_active(0) == loop.n_active(7) == sh.N
    loop.reset(x0, g0)
    loop.run(regroup=False)
    xr = O.run_loop(w, x0, g0, T, [8, 4, 2], counts, O.sigma_schedule(T, 1.0), sh.H, m=2,
                    regroup=False)
    d = _drift(host(loop.x), xr)
    print(f"tiny DiT with phase window m=2: x_T drift {d:.3e}")
    assert d <= 2e-2


def test_kernel_launch_counter():
    """The context counts the kernels it launches: per iteration schedule,
    embed, head and Euler, and per layer LN x2, QKV, attention + part-combine,
    out-proj, MLP up and down; re-grouping adds the cut search and assign (the
    Euler pass writes the scores)."""
    need_gpu()
    sh, T, counts, w, loop, x0, g0 = _setup()
    loop.reset(x0, g0)
    c0 = abi.hsa_kernel_launches(loop.ctx)
    loop.step(0)                               # no re-grouping before i = T / s_K = 2
    c1 = abi.hsa_kernel_launches(loop.ctx)
    loop.step(1)
    loop.step(2)                               # re-groups
    c3 = abi.hsa_kernel_launches(loop.ctx)
    abi.hsa_sync_check(loop.ctx)
    per_step = 4 + 8 * sh.L
    assert c1 - c0 == per_step
    assert c3 - c1 == 2 * per_step + 2
