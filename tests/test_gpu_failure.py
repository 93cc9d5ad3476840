"""Failure detection on the GPU without a fault: a bounded wait runs out.

hsa_selftest_timeout launches a kernel that waits on an mbarrier nothing
arrives at, through the same bounded wait every pipelined kernel uses.  The
wait must give up after its limit, the status must come back as
HSA_ERR_TIMEOUT through hsa_sync_check, and the context must keep working.
"""

import time

import numpy as np
import pytest

from gpu_util import dev, host, need_gpu, torch
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import abi, synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    need_gpu()
    N = 4096
    counts = synth.group_counts(N, (0.4, 0.3, 0.3))
    ctx = abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=40, budgets=[40, 20, 10], counts=counts)
    abi.hsa_sync_check(ctx)
    t0 = time.perf_counter()
    abi.hsa_selftest_timeout(ctx, 20000)          # 20 ms limit
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_sync_check(ctx)
    dt = time.perf_counter() - t0
    assert e.value.status == 6                    # HSA_ERR_TIMEOUT
    assert 0.015 <= dt < 5.0
    abi.hsa_sync_check(ctx)                        # flag cleared
    # the context still runs the path correctly
    g = synth.random_split(N, counts, 2)
    mask = torch.empty(N, dtype=torch.uint8, device="cuda")
    idx = torch.empty(N, dtype=torch.int32, device="cuda")
    n = abi.hsa_schedule(ctx, 4, dev(g), mask, idx)
    abi.hsa_sync_check(ctx)
    assert (host(idx)[:n] == O.active_index(O.active_mask(g, 4, 40, [40, 20, 10]))).all()


def test_selftest_rejects_bad_limit_on_host():
    need_gpu()
    ctx = abi.hsa_create(N=64, D=128, H=1, F=64, L=0, T=4, budgets=[4], counts=[64])
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_selftest_timeout(ctx, 0)
    assert e.value.status == 1
