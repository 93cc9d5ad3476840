"""Step-by-step checks of the GPU loop against what the pages fix, given the
GPU's own state (used by the loop tests at every size)."""

import numpy as np

from gpu_util import host
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import abi


def run_checked(loop, T, budgets, counts, g0, regroup=True, m=0):
    """Run the GPU loop one iteration at a time and check, at each one, what the
    pages fix given the GPU's own state ("Technical Summary: Heterogeneous Step
    Allocation (HSA) for Efficient Video Generation", 2.1): A_i is the schedule
    of the groups the iteration started from; a re-grouping scores the two
    cached velocities and assigns groups exactly as the oracle does.  Returns
    the number of re-groupings and how many group ids they changed."""
    r0 = O.regroup_from(T, budgets)
    g_prev = np.asarray(g0, dtype=np.uint8).copy()
    n_regroup = moved = 0
    for i in range(T):
        loop.step(i, regroup)
        abi.hsa_sync_check(loop.ctx)
        n = loop.n_active(i)
        want_idx = O.active_index(O.active_mask(g_prev, i, T, budgets, m))
        assert n == len(want_idx), i
        assert np.array_equal(host(loop.active_idx)[:n], want_idx), i
        g = host(loop.g)
        if regroup and r0 <= i < T - 1:
            vh, vp, sc = host(loop.v_hat), host(loop.v_hat_prev), host(loop.score)
            want = O.l1_relative_change(vp, vh)
            assert np.array_equal(sc.view(np.uint32), want.view(np.uint32)), i
            assert np.array_equal(g, O.assign_groups(sc, counts)), i
            n_regroup += 1
            moved += int((g != g_prev).sum())
        else:
            assert np.array_equal(g, g_prev), i
        g_prev = g
    return n_regroup, moved
