"""The HSA loop recorded as one CUDA graph (HsaLoop.capture) replays to the
same result as the eager loop, bit for bit, and replays again after reset()."""

import numpy as np
import pytest

from gpu_util import bf, dev, host, need_gpu
from token_sparse_denoising_layer_b200 import abi, synth

pytestmark = pytest.mark.gpu


def _loop(name, N=None, L=None):
    from token_sparse_denoising_layer_b200.loop import HsaLoop

    spec = synth.WORKLOADS[name]
    sh = spec["shape"]
    if N is not None:
        sh = synth.ModelShape(N=N, C=16, D=sh.D, H=sh.H, F=sh.F, L=L)
    counts = synth.group_counts(sh.N, spec["fractions"])
    w = synth.model_weights(sh, 12)
    layers = [tuple(bf(lw[k]) for k in ("w_qkv", "w_o", "w_1", "w_2")) for lw in w["layers"]]
    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]), spec["T"],
                   spec["budgets"], counts, shift=spec["shift"])
    x0 = synth.latent(sh.N, 16, 12)
    g0 = synth.random_split(sh.N, counts, 12)
    return loop, x0, g0


@pytest.mark.parametrize("name,N,L", [("tiny_dit", None, None), ("dit30_1536", 840, 1)])
def test_graph_replay_equals_eager_loop(name, N, L):
    need_gpu()
    loop, x0, g0 = _loop(name, N, L)
    loop.reset(x0, g0)
    n0 = abi.hsa_kernel_launches(loop.ctx)
    loop.run(regroup=True)
    eager_launches = abi.hsa_kernel_launches(loop.ctx) - n0
    abi.hsa_sync_check(loop.ctx)
    x_eager, g_eager = host(loop.x), host(loop.g)
    loop.capture(regroup=True)
    assert loop.graph_launches == eager_launches
    for _ in range(2):
        loop.reset(x0, g0)
        loop.replay()
        abi.hsa_sync_check(loop.ctx)
        assert np.array_equal(host(loop.x), x_eager)
        assert np.array_equal(host(loop.g), g_eager)
    loop.close()


def test_replay_needs_capture():
    need_gpu()
    loop, _, _ = _loop("tiny_dit")
    with pytest.raises(RuntimeError):
        loop.replay()
    loop.close()


def test_kernel_times_count_and_work_per_class():
    """hsa_time_kernels: one step of the tiny DiT with every launch timed. Per
    class the call counts follow the step's structure and the attention and
    GEMM work is the algorithmic FLOP of the step (4 a N D per attention, 2 M
    Ncols K per GEMM); reading clears the totals."""
    need_gpu()
    loop, x0, g0 = _loop("tiny_dit")
    loop.reset(x0, g0)
    abi.hsa_kernel_times(loop.ctx)
    abi.hsa_time_kernels(loop.ctx, True)
    loop.step(0)
    kt = abi.hsa_kernel_times(loop.ctx)
    abi.hsa_time_kernels(loop.ctx, False)
    abi.hsa_sync_check(loop.ctx)
    N, D, F, L = loop.N, loop.D, loop.F, loop.L
    a = loop.n_active(0)
    assert kt["attention"]["calls"] == L
    assert kt["gemm"]["calls"] == 4 * L
    assert kt["rows"]["calls"] == 2 * L + 2          # LN gathers, embed, head
    assert kt["tokens"]["calls"] == 2                # schedule, Euler
    assert kt["attention"]["work"] == L * 4.0 * a * N * D
    assert kt["gemm"]["work"] == L * 2.0 * a * (3 * D * D + D * D + 2 * D * F)
    for v in kt.values():
        assert v["ms"] > 0
    again = abi.hsa_kernel_times(loop.ctx)
    assert all(v["calls"] == 0 and v["ms"] == 0 for v in again.values())
    loop.close()
