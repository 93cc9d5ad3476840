"""hsa_select_groups_static: group selection for callers that cannot allocate.

Some callers cannot call cudaMalloc -- a host framework that owns all device
memory through its own pool, or a latency-critical loop that must not take
cudaMalloc's implicit device synchronisation -- so they cannot create a
context either.  This entry point keeps its scratch in a fixed static device
array instead.  Its group ids must equal those of the context-based
hsa_select_groups bit for bit, on consecutive calls that reuse the array.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import numpy as np
import pytest

from gpu_util import dev, host, need_gpu, torch
from token_sparse_denoising_layer_b200 import abi, synth

pytestmark = pytest.mark.gpu


def _reference_groups(vp_d, vc_d, N, budgets, counts):
    ctx = abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=budgets[0], budgets=budgets, counts=counts)
    score = torch.empty(N, dtype=torch.float32, device="cuda")
    g = torch.empty(N, dtype=torch.uint8, device="cuda")
    abi.hsa_select_groups(ctx, vp_d, vc_d, score, g)
    abi.hsa_sync_check(ctx)
    out = host(g).copy()
    ctx.close()
    return out


@pytest.mark.parametrize("calls", [
    # (N, budgets, fractions, seed) for two calls in a row
    [(32760, [40, 20, 10], (0.4, 0.3, 0.3), 11), (32760, [40, 20, 10], (0.4, 0.3, 0.3), 12)],
    [(75600, [40, 10], (0.25, 0.75), 13), (1001, [8, 4, 2, 1], (0.1, 0.2, 0.3, 0.4), 14)],
])
def test_static_select_matches_context_select(calls):
    need_gpu()
    for N, budgets, fr, seed in calls:
        counts = synth.group_counts(N, fr)
        vp, vc, _ = synth.velocity_pair(N, 16, seed)
        vp_d, vc_d = dev(vp), dev(vc)
        want = _reference_groups(vp_d, vc_d, N, budgets, counts)
        g = torch.full((N,), 255, dtype=torch.uint8, device="cuda")
        abi.hsa_select_groups_static(vp_d, vc_d, N, counts, g)
        torch.cuda.synchronize()
        assert (host(g) == want).all()
        assert [int((host(g) == k).sum()) for k in range(len(counts))] == counts


def test_static_select_rejects_sizes_beyond_its_scratch():
    need_gpu()
    N = abi.SELECT_STATIC_MAX_N + 1
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_select_groups_static(None, None, N, [N], None)
    assert e.value.status == 8
    assert "static scratch limit" in str(e.value)
