"""GPU parity of the per-token kernels against the oracle: schedule, selector, cached Euler.

Schedule, active index lists and group ids must be bit-exact; the score is
compared bit for bit with the oracle's float32 channel-order evaluation and
within 1e-6 of float64; the Euler update bit for bit with the oracle's
one-rounding-per-operation float32 form and within 1e-5 of float64.
"""

import numpy as np
import pytest

from gpu_util import EULER_TOL, dev, host, need_gpu, torch
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import abi, synth

pytestmark = pytest.mark.gpu

SIZES = [(1, [1], [1]), (37, [4, 2], [20, 17]), (4096, [40, 20, 10], None),
         (4097, [40, 20, 10], None), (32760, [40, 20, 10], None), (75600, [40, 10], None)]


def _ctx(N, budgets, counts=None, m=0):
    T = budgets[0]
    if counts is None:
        fr = [0.4, 0.3, 0.3] if len(budgets) == 3 else [0.25, 0.75] if len(budgets) == 2 else [1.0]
        counts = synth.group_counts(N, fr)
    return abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=T, budgets=budgets, counts=counts, m=m), counts


@pytest.mark.parametrize("N,budgets,counts", SIZES)
def test_schedule_bit_exact(N, budgets, counts):
    need_gpu()
    ctx, counts = _ctx(N, budgets, counts)
    T = budgets[0]
    g = synth.random_split(N, counts, 3)
    g_d = dev(g)
    mask_d = torch.empty(N, dtype=torch.uint8, device="cuda")
    idx_d = torch.full((N,), -1, dtype=torch.int32, device="cuda")
    n_d = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i in range(T):
        n_host = abi.hsa_schedule(ctx, i, g_d, mask_d, idx_d, n_d)
        mask = O.active_mask(g, i, T, budgets)
        idx = O.active_index(mask)
        assert n_host == len(idx) == O.n_active(i, T, budgets, counts)
        assert int(host(n_d)[0]) == len(idx)
        assert (host(mask_d) == mask.astype(np.uint8)).all()
        assert (host(idx_d)[: len(idx)] == idx).all()
    abi.hsa_sync_check(ctx)


def test_schedule_phase_window():
    need_gpu()
    N, budgets, m = 5000, [40, 20, 10], 3
    ctx, counts = _ctx(N, budgets, m=m)
    g = synth.random_split(N, counts, 4)
    g_d = dev(g)
    mask_d = torch.empty(N, dtype=torch.uint8, device="cuda")
    idx_d = torch.empty(N, dtype=torch.int32, device="cuda")
    for i in range(40):
        n = abi.hsa_schedule(ctx, i, g_d, mask_d, idx_d)
        idx = O.active_index(O.active_mask(g, i, 40, budgets, m))
        assert n == len(idx)
        assert (host(idx_d)[:n] == idx).all()


def test_schedule_bad_group_sets_flag():
    need_gpu()
    N = 64
    ctx, counts = _ctx(N, [4, 2], [32, 32])
    g = np.zeros(N, dtype=np.uint8)
    g[5] = 7  # >= K
    mask_d = torch.empty(N, dtype=torch.uint8, device="cuda")
    idx_d = torch.empty(N, dtype=torch.int32, device="cuda")
    abi.hsa_schedule(ctx, 0, dev(g), mask_d, idx_d)
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_sync_check(ctx)
    assert e.value.status == 7
    assert host(mask_d)[5] == 0
    abi.hsa_sync_check(ctx)  # flag cleared


@pytest.mark.parametrize("N", [1, 37, 4097, 32760, 75600])
@pytest.mark.parametrize("contiguous", [False, True])
def test_score_and_groups_bit_exact(N, contiguous):
    need_gpu()
    ctx, counts = _ctx(N, [40, 20, 10])
    vp, vc, low = synth.velocity_pair(N, 16, 5, contiguous=contiguous)
    score_d = torch.empty(N, dtype=torch.float32, device="cuda")
    g_d = torch.empty(N, dtype=torch.uint8, device="cuda")
    abi.hsa_select_groups(ctx, dev(vp), dev(vc), score_d, g_d)
    abi.hsa_sync_check(ctx)
    s_ref = O.l1_relative_change(vp, vc)
    s_gpu = host(score_d)
    assert (s_gpu.view(np.uint32) == s_ref.view(np.uint32)).all()
    s64 = O.l1_relative_change_f64(vp, vc)
    assert np.all(np.abs(s_gpu - s64) <= 1e-6 * np.abs(s64) + 1e-12)
    g_ref = O.assign_groups(s_ref, counts)
    assert (host(g_d) == g_ref).all()
    if N >= 100:
        assert (host(g_d)[low] == 2).all()


@pytest.mark.parametrize("N,ties", [(1, 0), (2, 1), (37, 3), (1000, 2), (32760, 5), (75600, 0), (75600, 7)])
def test_selection_from_shared_score_buffer(N, ties):
    """Given the same float32 score buffer, group ids are bit-exact (ties by index)."""
    need_gpu()
    for budgets, fr in (([40, 20, 10], (0.4, 0.3, 0.3)), ([40, 10], (0.25, 0.75)),
                        ([8, 4, 2, 1], (0.1, 0.2, 0.3, 0.4))):
        counts = synth.group_counts(N, fr)
        ctx = abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=budgets[0], budgets=budgets, counts=counts)
        s = synth.score_buffer(N, 9, n_tie_values=ties)
        g_d = torch.empty(N, dtype=torch.uint8, device="cuda")
        abi.hsa_select_from_score(ctx, dev(s), g_d)
        abi.hsa_sync_check(ctx)
        assert (host(g_d) == O.assign_groups(s, counts)).all()


def test_selection_empty_groups():
    need_gpu()
    N = 100
    counts = [100, 0, 0]
    ctx = abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=4, budgets=[4, 2, 1], counts=counts)
    s = synth.score_buffer(N, 1, n_tie_values=3)
    g_d = torch.empty(N, dtype=torch.uint8, device="cuda")
    abi.hsa_select_from_score(ctx, dev(s), g_d)
    assert (host(g_d) == 0).all()
    counts = [0, 0, 100]
    ctx = abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=4, budgets=[4, 2, 1], counts=counts)
    abi.hsa_select_from_score(ctx, dev(s), g_d)
    assert (host(g_d) == 2).all()


def test_selection_nan_sets_flag():
    need_gpu()
    N = 64
    ctx = abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=4, budgets=[4, 2], counts=[32, 32])
    s = synth.score_buffer(N, 2)
    s[3] = np.nan
    g_d = torch.empty(N, dtype=torch.uint8, device="cuda")
    abi.hsa_select_from_score(ctx, dev(s), g_d)
    with pytest.raises(abi.HsaError):
        abi.hsa_sync_check(ctx)


@pytest.mark.parametrize("N", [1, 255, 32760, 75600])
def test_euler_bit_exact(N):
    need_gpu()
    ctx, _ = _ctx(N, [40, 20, 10])
    r = synth.rng(N)
    x, vh, vp, vf = (r.standard_normal((N, 16), dtype=np.float32) for _ in range(4))
    mask = (r.random(N) < 0.45).astype(np.uint8)
    sig = O.sigma_schedule(40, 5.0)
    xd, vhd, vpd = dev(x), dev(vh), dev(vp)
    i = 17
    abi.hsa_euler_step(ctx, xd, vhd, vpd, dev(vf), dev(mask), sig[i], sig[i + 1])
    abi.hsa_sync_check(ctx)
    ex, eh, ep = O.euler_step_f32(x, vh, vp, vf, mask, sig[i], sig[i + 1])
    assert (host(xd).view(np.uint32) == ex.view(np.uint32)).all()
    assert (host(vhd) == eh).all() and (host(vpd) == ep).all()
    fx, _, _ = O.euler_step(x, vh, vp, vf, mask, sig[i], sig[i + 1])
    assert np.abs(host(xd) - fx).max() / np.abs(fx).max() <= EULER_TOL


@pytest.mark.parametrize("N", [1, 3, 255, 4097, 32760, 75600])
def test_euler_with_score_bit_exact(N):
    """The Euler pass that also scores the re-grouping: x and both caches as
    hsa_euler_step gives them, and the score bit for bit the oracle's float32
    L1 relative change of the updated (v_hat_prev, v_hat); a third of the tokens
    are active, the rest score from caches they did not touch this step."""
    need_gpu()
    ctx, counts = _ctx(N, [40, 20, 10])
    r = synth.rng(N + 7)
    x, vh, vp, vf = (r.standard_normal((N, 16), dtype=np.float32) for _ in range(4))
    vp[::5] = vh[::5] + np.float32(0.01) * vp[::5]          # a low-change region
    mask = (r.random(N) < 0.35).astype(np.uint8)
    sig = O.sigma_schedule(40, 5.0)
    i = 23
    xd, vhd, vpd = dev(x), dev(vh), dev(vp)
    score = torch.full((N,), -1.0, dtype=torch.float32, device="cuda")
    abi.hsa_euler_step_score(ctx, xd, vhd, vpd, dev(vf), dev(mask), sig[i], sig[i + 1], score)
    abi.hsa_sync_check(ctx)
    ex, eh, ep = O.euler_step_f32(x, vh, vp, vf, mask, sig[i], sig[i + 1])
    assert (host(xd).view(np.uint32) == ex.view(np.uint32)).all()
    assert (host(vhd) == eh).all() and (host(vpd) == ep).all()
    want = O.l1_relative_change(ep, eh)
    assert (host(score).view(np.uint32) == want.view(np.uint32)).all()
    # the same buffer through the standalone score kernel
    s2 = torch.empty((N,), dtype=torch.float32, device="cuda")
    abi.hsa_score(ctx, vpd, vhd, s2)
    assert (host(s2).view(np.uint32) == want.view(np.uint32)).all()
    ctx.close()


def test_euler_all_skipped_and_closed_form():
    """Mask all zero: caches untouched; T steps telescope to x0 + v (sigma_T - sigma_0)."""
    need_gpu()
    N, T = 32760, 40
    ctx, _ = _ctx(N, [40, 20, 10])
    r = synth.rng(1)
    x0 = r.standard_normal((N, 16), dtype=np.float32)
    v = r.standard_normal((N, 16), dtype=np.float32)
    sig = O.sigma_schedule(T, 5.0)
    xd, vhd, vpd = dev(x0), dev(v), dev(np.zeros_like(v))
    z = dev(np.zeros_like(v))
    m0 = dev(np.zeros(N, dtype=np.uint8))
    for i in range(T):
        abi.hsa_euler_step(ctx, xd, vhd, vpd, z, m0, sig[i], sig[i + 1])
    assert (host(vhd) == v).all() and (host(vpd) == 0).all()
    closed = x0.astype(np.float64) + v.astype(np.float64) * (float(sig[T]) - float(sig[0]))
    # T float32 steps: each rounds once in the product and once in the sum
    assert np.abs(host(xd) - closed).max() <= 2 * T * 2.0 ** -24 * (np.abs(x0).max() + np.abs(v).max())
