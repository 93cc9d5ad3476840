"""Seeded synthetic inputs for the HSA denoising step.

This module only draws random numbers and fixes shapes.  It holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can be fed from it
without sharing any computation.  Every array is produced on the host with
numpy's PCG64 generator from an explicit seed, so the same call gives the same
bytes on every machine.

Workloads follow the shapes of the Heterogeneous Step Allocation (HSA) method
("Not All Tokens Need 40 Steps: Heterogeneous Step Allocation in Diffusion
Transformers for Efficient Video Generation"): a video latent of t x h x w
tokens with 16 channels, a diffusion-transformer stack of pre-LN blocks with
random N(0, 1/fan_in) weights, and K token groups with step budgets s_k | T.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Sequence

import numpy as np

__all__ = [
    "ModelShape",
    "WORKLOADS",
    "group_counts",
    "bf16_round",
    "rng",
    "latent",
    "random_split",
    "velocity_pair",
    "layer_weights",
    "model_weights",
    "hidden_rows",
    "stale_kv",
    "random_active_set",
    "attention_inputs",
    "score_buffer",
    "modulation",
    "cross_attention_weights",
]


@dataclasses.dataclass(frozen=True)
class ModelShape:
    """Shape of a diffusion-transformer workload.

    N tokens, C latent channels, D hidden, H heads of head_dim d = D / H,
    F MLP width, L layers.
    """

    N: int
    C: int
    D: int
    H: int
    F: int
    L: int

    @property
    def d(self) -> int:
        return self.D // self.H


# Named workloads.  Sizes follow the latent grids they describe.
WORKLOADS: Dict[str, dict] = {
    # 4x8x8 latent, 2 layers, T=8 on a linear sigma schedule, budgets {8,4} at 50/50.
    "tiny_dit": dict(shape=ModelShape(N=256, C=16, D=128, H=2, F=512, L=2),
                     T=8, budgets=(8, 4), fractions=(0.5, 0.5), shift=1.0, seed=0),
    # Scheduler / selector / cached-Euler standalone, 21x30x52 and 21x45x80 latents.
    "select_euler_32760": dict(N=32760, C=16, T=40, budgets=(40, 20, 10),
                               fractions=(0.4, 0.3, 0.3), shift=5.0, seed=0),
    "select_euler_75600": dict(N=75600, C=16, T=40, budgets=(40, 20, 10),
                               fractions=(0.4, 0.3, 0.3), shift=5.0, seed=0),
    # Single bf16 DiT layer, hidden 1536, 12 x 128 heads, MLP 4x.
    "layer_1536": dict(shape=ModelShape(N=32760, C=16, D=1536, H=12, F=6144, L=1),
                       fractions_active=(1.0, 0.5, 0.25, 0.1), seed=0),
    # Full HSA loop, 30-layer DiT, hidden 1536, MLP 8960, 21x30x52 latent.
    "dit30_1536": dict(shape=ModelShape(N=32760, C=16, D=1536, H=12, F=8960, L=30),
                       T=40, budgets=(40, 20, 10), fractions=(0.4, 0.3, 0.3),
                       shift=5.0, seed=0),
    # Large-shape loop, 40-layer DiT, hidden 5120, MLP 13824, 21x45x80 latent.
    "dit40_5120": dict(shape=ModelShape(N=75600, C=16, D=5120, H=40, F=13824, L=40),
                       T=40, budgets=(40, 10), fractions=(0.25, 0.75), shift=5.0, seed=0),
}


def group_counts(N: int, fractions: Sequence[float]) -> List[int]:
    """Token count per group: floor(f_k * N) for k >= 2, the rest to group 1."""
    rest = [int(np.floor(f * N + 1e-9)) for f in fractions[1:]]
    return [N - sum(rest)] + rest


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even), returned as float32.

    Used to make synthetic weights and caches that are exactly representable in
    bf16, so the oracle and the GPU read identical values.
    """
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16 << 16
    return (u.astype(np.uint32)).view(np.float32).reshape(f.shape)


def latent(N: int, C: int, seed: int) -> np.ndarray:
    """Initial latent x ~ N(0, 1), float32 [N, C]."""
    return rng(seed).standard_normal((N, C), dtype=np.float32)


def random_split(N: int, counts: Sequence[int], seed: int) -> np.ndarray:
    """Initial group ids: a seeded random permutation cut at the group counts.

    The first counts[0] tokens of the permutation go to group 0 (full budget),
    the next counts[1] to group 1, and so on.  Returns uint8 [N].
    """
    assert sum(counts) == N
    perm = rng(seed + 7919).permutation(N)
    g = np.empty(N, dtype=np.uint8)
    start = 0
    for k, c in enumerate(counts):
        g[perm[start:start + c]] = k
        start += c
    return g


def velocity_pair(N: int, C: int, seed: int, low_frac: float = 0.3,
                  contiguous: bool = False):
    """v_prev, v_cur ~ N(0,1) float32 [N, C] with a low-change region.

    floor(low_frac * N) tokens (a seeded random subset, or the first ones in
    raster order when ``contiguous``) get v_cur = v_prev + 0.01 * z.  Returns
    (v_prev, v_cur, low_set) where low_set is a bool [N] marking that region.
    """
    r = rng(seed)
    v_prev = r.standard_normal((N, C), dtype=np.float32)
    v_cur = r.standard_normal((N, C), dtype=np.float32)
    n_low = int(np.floor(low_frac * N + 1e-9))
    if contiguous:
        low = np.arange(n_low)
    else:
        low = r.permutation(N)[:n_low]
    z = r.standard_normal((n_low, C), dtype=np.float32)
    v_cur[low] = v_prev[low] + np.float32(0.01) * z
    low_set = np.zeros(N, dtype=bool)
    low_set[low] = True
    return v_prev, v_cur, low_set


def _linear(r: np.random.Generator, out_f: int, in_f: int) -> np.ndarray:
    w = r.standard_normal((out_f, in_f), dtype=np.float32) * np.float32(1.0 / np.sqrt(in_f))
    return w


def layer_weights(D: int, F: int, seed: int) -> Dict[str, np.ndarray]:
    """One block's weights in Linear layout [out, in], bf16-representable float32.

    w_qkv [3D, D] (rows 0..D-1 give Q, D..2D-1 give K, 2D..3D-1 give V),
    w_o [D, D], w_1 [F, D], w_2 [D, F].  Entries ~ N(0, 1/fan_in).
    """
    r = rng(seed)
    return {
        "w_qkv": bf16_round(_linear(r, 3 * D, D)),
        "w_o": bf16_round(_linear(r, D, D)),
        "w_1": bf16_round(_linear(r, F, D)),
        "w_2": bf16_round(_linear(r, D, F)),
    }


def model_weights(shape: ModelShape, seed: int) -> Dict[str, object]:
    """Embed [D, C], per-layer block weights, and velocity head [C, D].

    The embed and head stay float32 (they are small); block weights are bf16
    values.
    """
    r = rng(seed + 1)
    w_in = _linear(r, shape.D, shape.C)
    w_head = _linear(r, shape.C, shape.D)
    layers = [layer_weights(shape.D, shape.F, seed + 100 + l) for l in range(shape.L)]
    return {"w_in": w_in, "w_head": w_head, "layers": layers}


def hidden_rows(N: int, D: int, seed: int) -> np.ndarray:
    """Hidden state x ~ N(0, 1), float32 [N, D]."""
    return rng(seed + 11).standard_normal((N, D), dtype=np.float32)


def stale_kv(N: int, D: int, seed: int):
    """Pre-filled stale K and V caches ~ N(0, 1), bf16 values as float32 [N, D]."""
    r = rng(seed + 13)
    k = bf16_round(r.standard_normal((N, D), dtype=np.float32))
    v = bf16_round(r.standard_normal((N, D), dtype=np.float32))
    return k, v


def random_active_set(N: int, a: int, seed: int) -> np.ndarray:
    """A seeded random subset of a token indices, ascending, int32."""
    idx = rng(seed + 17).permutation(N)[:a]
    return np.sort(idx).astype(np.int32)


def attention_inputs(a: int, N: int, D: int, seed: int, q_scale: float = 1.0):
    """Q [a, D] and K, V caches [N, D]: bf16 values as float32.

    ``q_scale`` widens the query distribution so the softmax is peaked, which
    makes a wrong scale or a wrong key order visible in the output.
    """
    r = rng(seed + 19)
    q = bf16_round(r.standard_normal((a, D), dtype=np.float32) * np.float32(q_scale))
    k = bf16_round(r.standard_normal((N, D), dtype=np.float32))
    v = bf16_round(r.standard_normal((N, D), dtype=np.float32))
    return q, k, v


def score_buffer(N: int, seed: int, n_tie_values: int = 0) -> np.ndarray:
    """A non-negative float32 score per token, for testing the ranking alone.

    With ``n_tie_values`` > 0 the scores are drawn from that many distinct
    values only, so many tokens tie and the index tie-break decides.
    """
    r = rng(seed + 23)
    if n_tie_values > 0:
        vals = np.abs(r.standard_normal(n_tie_values).astype(np.float32))
        s = vals[r.integers(0, n_tie_values, N)]
    else:
        s = np.abs(r.standard_normal(N).astype(np.float32))
    s[r.integers(0, N, max(1, N // 100))] = 0.0
    return s.astype(np.float32)


def device_layer_weights(D: int, F: int, seed: int, device="cuda"):
    """Block weights ~ N(0, 1/fan_in) drawn on the device (torch Philox), bf16.

    For workloads whose weights are too large to draw on the host quickly
    (tens of layers at D = 1536).  Returns (w_qkv, w_o, w_1, w_2).
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def lin(o, i):
        return (torch.randn((o, i), generator=g, device=device, dtype=torch.float32)
                * (1.0 / np.sqrt(i))).to(torch.bfloat16)

    return lin(3 * D, D), lin(D, D), lin(F, D), lin(D, F)


def modulation(D: int, seed: int, spread: float = 0.5) -> np.ndarray:
    """Timestep modulation vectors [6, D] float32: (shift, scale, gate) for the
    attention branch, then for the MLP branch; shifts/scales ~ spread*N(0,1),
    gates ~ 1 + spread*N(0,1)."""
    r = rng(seed + 29)
    m = (r.standard_normal((6, D)) * spread).astype(np.float32)
    m[2] += 1.0
    m[5] += 1.0
    return m


def cross_attention_weights(D: int, n_txt: int, seed: int) -> Dict[str, np.ndarray]:
    """Text cross-attention: w_q, w_o [D, D] ~ N(0, 1/D) and the text tokens'
    keys and values k_txt, v_txt [n_txt, D] ~ N(0, 1), all bf16 values as float32."""
    r = rng(seed + 31)
    return {"w_q": bf16_round(_linear(r, D, D)), "w_o": bf16_round(_linear(r, D, D)),
            "k_txt": bf16_round(r.standard_normal((n_txt, D), dtype=np.float32)),
            "v_txt": bf16_round(r.standard_normal((n_txt, D), dtype=np.float32))}
