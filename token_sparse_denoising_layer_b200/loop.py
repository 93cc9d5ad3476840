"""Host side of the HSA denoising loop: device state, noise levels, one call per step.

Each global iteration is one ``hsa_step`` call into libhsa (schedule -> embed
-> every layer on the active set -> head -> cached Euler -> re-grouping); this
module only allocates the buffers and walks i = 0..T-1.  Method: "Technical
Summary: Heterogeneous Step Allocation (HSA) for Efficient Video Generation",
sections 2.1-2.3.
"""

from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from . import abi


def sigma_schedule(T: int, shift: float = 1.0) -> np.ndarray:
    """Noise levels sigma_0..sigma_T (float32): linear from 1 to 0, then the
    flow-matching timestep shift s*sigma / (1 + (s-1)*sigma)."""
    s = 1.0 - np.arange(T + 1, dtype=np.float64) / T
    return (shift * s / (1.0 + (shift - 1.0) * s)).astype(np.float32)


class HsaLoop:
    """Device-resident model and loop state for one HSA sampling run.

    ``layers`` holds, per block, the bf16 CUDA tensors (w_qkv, w_o, w_1, w_2);
    ``w_in`` [D, C] and ``w_head`` [C, D] are float32 CUDA tensors.
    """

    def __init__(self, N: int, D: int, H: int, F: int, layers, w_in, w_head, T: int,
                 budgets: Sequence[int], counts: Sequence[int], shift: float = 1.0, m: int = 0,
                 stream=None):
        import torch

        self.torch = torch
        self.N, self.D, self.H, self.F, self.L = N, D, H, F, len(layers)
        self.T, self.budgets, self.counts = T, list(budgets), list(counts)
        self.ctx = abi.hsa_create(N=N, D=D, H=H, F=F, L=self.L, T=T, budgets=budgets,
                                  counts=counts, m=m, stream=stream)
        self._stream = stream
        self.graph = None
        self.graph_launches = 0
        dev = "cuda"
        f32 = dict(dtype=torch.float32, device=dev)
        self.x = torch.zeros((N, 16), **f32)
        self.v_hat = torch.zeros((N, 16), **f32)
        self.v_hat_prev = torch.zeros((N, 16), **f32)
        self.v_fresh = torch.zeros((N, 16), **f32)
        self.score = torch.zeros((N,), **f32)
        self.g = torch.zeros((N,), dtype=torch.uint8, device=dev)
        self.mask = torch.zeros((N,), dtype=torch.uint8, device=dev)
        self.active_idx = torch.zeros((N,), dtype=torch.int32, device=dev)
        self.h = torch.zeros((N, D), **f32)
        self.k_cache = [torch.zeros((N, D), dtype=torch.bfloat16, device=dev) for _ in layers]
        self.v_cache = [torch.zeros((N, D), dtype=torch.bfloat16, device=dev) for _ in layers]
        self.sigmas = sigma_schedule(T, shift)
        self.model = abi.ModelBinding(w_in, w_head, layers, self.x, self.v_hat, self.v_hat_prev,
                                      self.v_fresh, self.score, self.g, self.mask,
                                      self.active_idx, self.h, self.k_cache, self.v_cache)

    def reset(self, x0, g0) -> None:
        """Start a new run from latent x0 [N, 16] and group ids g0 [N] (tensors or arrays)."""
        t = self.torch
        self.x.copy_(t.as_tensor(np.asarray(x0) if not t.is_tensor(x0) else x0))
        self.g.copy_(t.as_tensor(np.asarray(g0) if not t.is_tensor(g0) else g0))
        for buf in (self.v_hat, self.v_hat_prev, self.v_fresh, self.score):
            buf.zero_()

    def n_active(self, i: int) -> int:
        return abi.hsa_n_active(self.ctx, i)

    def step(self, i: int, regroup: bool = True, cond: "Optional[abi.StepCond]" = None) -> None:
        """Iteration i; ``cond`` carries conditioned blocks' modulation and
        cross-attention for this iteration (abi.StepCond), or None."""
        if cond is None:
            abi.hsa_step(self.ctx, self.model, i, float(self.sigmas[i]),
                         float(self.sigmas[i + 1]), regroup)
        else:
            abi.hsa_step_cond(self.ctx, self.model, cond, i, float(self.sigmas[i]),
                              float(self.sigmas[i + 1]), regroup)

    def run(self, regroup: bool = True, stop: Optional[int] = None):
        for i in range(self.T if stop is None else stop):
            self.step(i, regroup)
        return self.x

    def capture(self, regroup: bool = True) -> None:
        """Record the whole loop, i = 0..T-1, as one CUDA graph.

        Every step's launch shape is fixed by the host (|A_i| follows from the
        group counts), so the T steps replay as recorded; the graph reads and
        writes this loop's buffers in place.  Call after at least one eager
        step (first calls set kernel attributes), and reset() before replay()."""
        t = self.torch
        t.cuda.synchronize()
        side = t.cuda.Stream()
        g = t.cuda.CUDAGraph()
        n0 = abi.hsa_kernel_launches(self.ctx)
        abi.hsa_set_stream(self.ctx, side)
        try:
            with t.cuda.graph(g, stream=side):
                for i in range(self.T):
                    self.step(i, regroup)
        finally:
            abi.hsa_set_stream(self.ctx, self._stream)
        self.graph_launches = abi.hsa_kernel_launches(self.ctx) - n0
        self.graph = g

    def replay(self) -> None:
        """Run the recorded loop on the current stream."""
        if self.graph is None:
            raise RuntimeError("capture() first")
        self.graph.replay()

    def close(self) -> None:
        self.graph = None
        self.ctx.close()
