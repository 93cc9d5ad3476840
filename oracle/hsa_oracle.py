"""CPU oracle for the Heterogeneous Step Allocation (HSA) denoising step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this file; only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline do.  It shares no code with the CUDA path.

It is a plain, slow, step-by-step restatement of the method, in float64 numpy
unless a step's result is an integer decision (see ``l1_relative_change``).
Each function cites the passage it follows.  Sources:

  [TS]  "Technical Summary: Heterogeneous Step Allocation (HSA) for Efficient
        Video Generation" (gist.science/paper/2605.06892), sections 2.1-2.4.
  [ABS] "Not All Tokens Need 40 Steps: Heterogeneous Step Allocation in
        Diffusion Transformers for Efficient Video Generation", abstract.

Where the pages are silent, the plainest reading is taken and named in the
docstring ("reading: ...").  Parity status per function:
  pinned   - checked in tests against closed forms, brute force or invariants
  readings - the shift form of ``sigma_schedule`` and the re-grouping cadence
             in ``run_loop`` are conventions the pages leave open; the code
             is pinned to them (the shift by its odds identity, the cadence
             by its first re-grouping step).
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "check_budgets", "strides", "active_mask", "active_index", "n_active",
    "l1_relative_change", "l1_relative_change_f64", "rank_keys_order",
    "assign_groups", "sigma_schedule", "linear", "layer_norm", "gelu", "bf16",
    "attention", "layer_forward", "embed", "head", "euler_step",
    "euler_step_f32", "regroup_from", "run_loop", "dense_loop",
]

LN_EPS = 1e-5          # reading: LayerNorm without affine, eps 1e-5
SCORE_EPS = 1e-6       # reading: eps in the L1 relative change denominator


# --------------------------------------------------------------------------
# [TS] 2.1 Token Partitioning and Scheduling
# --------------------------------------------------------------------------

def check_budgets(T: int, budgets: Sequence[int], counts: Optional[Sequence[int]] = None,
                  N: Optional[int] = None) -> None:
    """Validate a group layout ([TS] 2.1).

    Every budget s_k divides T; the baseline group has s_1 = T.  Reading: the
    budgets are strictly decreasing (group 1 is the full group, later groups
    get fewer steps) and the group counts sum to N.
    """
    if T <= 0 or len(budgets) == 0:
        raise ValueError("T and K must be positive")
    if budgets[0] != T:
        raise ValueError("baseline group must have s_1 = T")
    for a, b in zip(budgets, budgets[1:]):
        if not b < a:
            raise ValueError("budgets must be strictly decreasing")
    for s in budgets:
        if s <= 0 or T % s != 0:
            raise ValueError(f"budget {s} does not divide T={T}")
    if counts is not None:
        if len(counts) != len(budgets) or any(c < 0 for c in counts):
            raise ValueError("one non-negative count per group")
        if N is not None and sum(counts) != N:
            raise ValueError("group counts must sum to N")


def strides(T: int, budgets: Sequence[int]) -> List[int]:
    """tau_k = T / s_k, the spacing between a group's active iterations ([TS] 2.1)."""
    return [T // s for s in budgets]


def active_mask(g: np.ndarray, i: int, T: int, budgets: Sequence[int], m: int = 0) -> np.ndarray:
    """Active predicate of every token at global iteration i ([TS] 2.1, 2.4).

    A token of group k is active iff i mod (T/s_k) == 0.  Reading: i runs
    0..T-1.  Phase-aware window ([TS] 2.4): the first m and last m iterations
    are full passes for all tokens.
    """
    tau = np.asarray(strides(T, budgets), dtype=np.int64)
    on = (i % tau[g.astype(np.int64)]) == 0
    if m > 0 and (i < m or i >= T - m):
        on = np.ones_like(on)
    return on


def active_index(mask: np.ndarray) -> np.ndarray:
    """A_i as ascending int32 token indices (reading: ascending order)."""
    return np.flatnonzero(mask).astype(np.int32)


def n_active(i: int, T: int, budgets: Sequence[int], counts: Sequence[int], m: int = 0) -> int:
    """|A_i| from the group sizes alone ([TS] 2.1): sum of n_k over active groups."""
    if m > 0 and (i < m or i >= T - m):
        return int(sum(counts))
    return int(sum(c for c, t in zip(counts, strides(T, budgets)) if i % t == 0))


def l1_relative_change(v_prev: np.ndarray, v_cur: np.ndarray, eps: float = SCORE_EPS) -> np.ndarray:
    """Per-token L1 relative change of the velocity prediction ([TS] 2.1, Dynamic Selection).

    r_n = sum_c |v_cur - v_prev| / (sum_c |v_prev| + eps).

    The score decides an integer (the group), so it is evaluated in the
    kernel's precision: float32, each sum taken in channel order 0..C-1, one
    IEEE division.  ``l1_relative_change_f64`` is the same quantity in float64.
    """
    vp = np.asarray(v_prev, dtype=np.float32)
    vc = np.asarray(v_cur, dtype=np.float32)
    num = np.zeros(vp.shape[0], dtype=np.float32)
    den = np.zeros(vp.shape[0], dtype=np.float32)
    for c in range(vp.shape[1]):
        num = (num + np.abs(vc[:, c] - vp[:, c])).astype(np.float32)
        den = (den + np.abs(vp[:, c])).astype(np.float32)
    den = (den + np.float32(eps)).astype(np.float32)
    r = (num / den).astype(np.float32)
    return r + np.float32(0.0)    # maps -0.0 to +0.0


def l1_relative_change_f64(v_prev: np.ndarray, v_cur: np.ndarray, eps: float = SCORE_EPS) -> np.ndarray:
    """The same score as ``l1_relative_change`` in float64."""
    vp = np.asarray(v_prev, dtype=np.float64)
    vc = np.asarray(v_cur, dtype=np.float64)
    return np.abs(vc - vp).sum(axis=1) / (np.abs(vp).sum(axis=1) + eps)


def rank_keys_order(score: np.ndarray) -> np.ndarray:
    """Token order by (score descending, index ascending).

    Reading: faster-changing tokens rank first; ties go to the lower index.
    """
    s = np.asarray(score, dtype=np.float32)
    if not np.all(np.isfinite(s)) or np.any(s < 0):
        raise ValueError("scores must be finite and non-negative")
    n = np.arange(s.shape[0])
    return np.lexsort((n, -s.astype(np.float64)))


def assign_groups(score: np.ndarray, counts: Sequence[int]) -> np.ndarray:
    """Dynamic Token Selection ([TS] 2.1): group ids from a score buffer.

    Slow-evolving tokens (low relative change) get the reduced budgets.
    Reading: the counts[0] highest-scoring tokens go to group 0 (budget T),
    the next counts[1] to group 1, and so on; ties broken by token index.
    """
    order = rank_keys_order(score)
    g = np.empty(order.shape[0], dtype=np.uint8)
    start = 0
    for k, c in enumerate(counts):
        g[order[start:start + c]] = k
        start += c
    return g


# --------------------------------------------------------------------------
# Sampler pieces
# --------------------------------------------------------------------------

def sigma_schedule(T: int, shift: float = 1.0) -> np.ndarray:
    """Noise levels sigma_0..sigma_T as float32.

    Reading: linear sigma_j = 1 - j/T, then the flow-matching timestep shift
    sigma' = s*sigma / (1 + (s-1)*sigma); computed in float64, rounded to float32.
    """
    j = np.arange(T + 1, dtype=np.float64)
    s = 1.0 - j / T
    s = shift * s / (1.0 + (shift - 1.0) * s)
    return s.astype(np.float32)


def bf16(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), returned as float64.

    Used only when emulating the storage points of a bf16 model.
    """
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64).reshape(f.shape)


def linear(a: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Active-row linear map a w^T with w in Linear layout [out, in] ([TS] 2.2)."""
    return np.asarray(a, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


def layer_norm(x: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """LayerNorm over the last axis, no affine (reading: pre-LN block, eps 1e-5)."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def gelu(x: np.ndarray) -> np.ndarray:
    """GELU, exact erf form: x * Phi(x)."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


# --------------------------------------------------------------------------
# [TS] 2.2 KV-Cache Synchronization
# --------------------------------------------------------------------------

def attention(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, H: int,
              emulate_bf16: bool = False) -> np.ndarray:
    """Full-context attention of the active queries ([TS] 2.2, step 3).

    q [a, D] attends, per head, to all N cached keys/values [N, D]:
    O = softmax(q k^T / sqrt(d)) v.  Cost O(|A_i| * N) ([TS] 2.2, step 4).
    With ``emulate_bf16`` the probabilities are rounded to bf16 before the
    product with V and O is rounded to bf16, as a bf16 kernel stores them.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(k_cache, dtype=np.float64)
    V = np.asarray(v_cache, dtype=np.float64)
    a, D = q.shape
    d = D // H
    out = np.empty((a, D), dtype=np.float64)
    for h in range(H):
        sl = slice(h * d, (h + 1) * d)
        s = (q[:, sl] @ K[:, sl].T) / math.sqrt(d)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        l = p.sum(axis=1, keepdims=True)
        if emulate_bf16:
            p = bf16(p)
        out[:, sl] = (p @ V[:, sl]) / l
    if emulate_bf16:
        out = bf16(out)
    return out


def layer_forward(w: Dict[str, np.ndarray], x: np.ndarray, idx: np.ndarray,
                  k_cache: np.ndarray, v_cache: np.ndarray, H: int,
                  emulate_bf16: bool = False, trace: Optional[dict] = None,
                  mod: Optional[np.ndarray] = None, cross: Optional[dict] = None) -> None:
    """One transformer block on the active set only ([TS] 2.2), in place.

    1. Only A_i goes through the QKV projection (step 1).
    2. Its fresh K, V rows overwrite the stale rows of this layer's cache (step 2).
    3. Its queries attend to all N cached rows (step 3).
    4. Out-projection and MLP run on A_i only; skipped tokens get no query and no
       feed-forward (step 4).  Results are added back into rows idx of x.

    Reading (the pages give no architecture): pre-LN residual block
    x += W_o Attn(LN(x)); x += W_2 GELU(W_1 LN(x)); no biases.  Weights are in
    Linear layout [out, in].  x is float [N, D]; k_cache, v_cache are float
    [N, D] (H heads of d = D/H).  ``emulate_bf16`` rounds at the points a bf16
    kernel stores: LN outputs, Q/K/V, probabilities, attention output, GELU output.

    Conditioning of a real video DiT (reading; [TS] 2.2 step 4 says skipped
    tokens incur no cross-attention, so both act on A_i only):
    ``mod`` [6, D] = (shift_a, scale_a, gate_a, shift_m, scale_m, gate_m), the
    timestep modulation shared by all active tokens at this iteration:
    LN(x)*(1 + scale) + shift before the attention / MLP branch, and the branch
    output multiplied by its gate.  ``cross`` = {w_q, w_o, k_txt, v_txt}: after
    self-attention, x += W_oc Attn(LN(x) W_qc^T, k_txt, v_txt) against the text
    tokens' keys and values (no cache: they are fixed for the whole run).
    """
    rb = bf16 if emulate_bf16 else (lambda t: t)
    D = x.shape[1]
    xa = np.asarray(x[idx], dtype=np.float64)
    m = None if mod is None else np.asarray(mod, dtype=np.float64)
    u = layer_norm(xa)
    if m is not None:
        u = u * (1.0 + m[1]) + m[0]
    u = rb(u)
    qkv = u @ np.asarray(w["w_qkv"], dtype=np.float64).T
    q = rb(qkv[:, :D])
    k = rb(qkv[:, D:2 * D])
    v = rb(qkv[:, 2 * D:])
    k_cache[idx] = k
    v_cache[idx] = v
    o = attention(q, k_cache, v_cache, H, emulate_bf16)
    branch = o @ np.asarray(w["w_o"], dtype=np.float64).T
    xa = xa + (branch if m is None else m[2] * branch)
    oc = None
    if cross is not None:
        uc = rb(layer_norm(xa))
        qc = rb(uc @ np.asarray(cross["w_q"], dtype=np.float64).T)
        oc = attention(qc, cross["k_txt"], cross["v_txt"], H, emulate_bf16)
        xa = xa + oc @ np.asarray(cross["w_o"], dtype=np.float64).T
    u2 = layer_norm(xa)
    if m is not None:
        u2 = u2 * (1.0 + m[4]) + m[3]
    u2 = rb(u2)
    hmid = rb(gelu(u2 @ np.asarray(w["w_1"], dtype=np.float64).T))
    branch = hmid @ np.asarray(w["w_2"], dtype=np.float64).T
    xa = xa + (branch if m is None else m[5] * branch)
    x[idx] = xa
    if trace is not None:
        trace.update(q=q, k=k, v=v, o=o, u=u, u2=u2, hmid=hmid, oc=oc)


def embed(w_in: np.ndarray, x_lat: np.ndarray) -> np.ndarray:
    """Latent rows [a, C] -> hidden rows [a, D] (reading: linear patch embed, no bias)."""
    return np.asarray(x_lat, dtype=np.float64) @ np.asarray(w_in, dtype=np.float64).T


def head(w_head: np.ndarray, h: np.ndarray) -> np.ndarray:
    """Hidden rows [a, D] -> velocity rows [a, C] (reading: final LN, then linear)."""
    return layer_norm(h) @ np.asarray(w_head, dtype=np.float64).T


# --------------------------------------------------------------------------
# [TS] 2.3 Cached Euler Update
# --------------------------------------------------------------------------

def euler_step(x, v_hat, v_hat_prev, v_fresh, mask, sigma_i: float, sigma_next: float):
    """Cached Euler update over all N tokens ([TS] 2.3), float64.

    Every token keeps the velocity of its latest active step (v_hat).  Active
    tokens take their fresh velocity, skipped tokens reuse the cached one, and
    all advance by the same increment sigma_{i+1} - sigma_i.  Reading: v_hat_prev
    keeps the velocity before the latest one (the selector compares the two).
    Returns new (x, v_hat, v_hat_prev).
    """
    mk = np.asarray(mask, dtype=bool)[:, None]
    v_hat = np.asarray(v_hat, dtype=np.float64)
    v_hat_prev = np.asarray(v_hat_prev, dtype=np.float64)
    v_fresh = np.asarray(v_fresh, dtype=np.float64)
    new_prev = np.where(mk, v_hat, v_hat_prev)
    new_hat = np.where(mk, v_fresh, v_hat)
    dsig = float(sigma_next) - float(sigma_i)
    new_x = np.asarray(x, dtype=np.float64) + dsig * new_hat
    return new_x, new_hat, new_prev


def euler_step_f32(x, v_hat, v_hat_prev, v_fresh, mask, sigma_i, sigma_next):
    """The cached Euler update evaluated in float32, one rounding per operation.

    d = fl(sigma_next - sigma_i); x' = fl(x + fl(d * v)).  Same definition as
    ``euler_step``; this form lets a float32 kernel be compared bit for bit.
    """
    mk = np.asarray(mask, dtype=bool)[:, None]
    new_prev = np.where(mk, v_hat, v_hat_prev).astype(np.float32)
    new_hat = np.where(mk, v_fresh, v_hat).astype(np.float32)
    d = np.float32(np.float32(sigma_next) - np.float32(sigma_i))
    prod = (d * new_hat).astype(np.float32)
    new_x = (np.asarray(x, dtype=np.float32) + prod).astype(np.float32)
    return new_x, new_hat, new_prev


# --------------------------------------------------------------------------
# The denoising loop
# --------------------------------------------------------------------------

def regroup_from(T: int, budgets: Sequence[int]) -> int:
    """First iteration after which groups are re-selected (reading, unpinned).

    After iteration T/s_K every token has been active at least twice, so both
    cached velocities exist and every score is defined.
    """
    return T // min(budgets)


def run_loop(weights: dict, x0: np.ndarray, g0: np.ndarray, T: int,
             budgets: Sequence[int], counts: Sequence[int], sigmas: np.ndarray,
             H: int, m: int = 0, regroup: bool = True, emulate_bf16: bool = False,
             log: Optional[list] = None, mods=None, cross=None) -> np.ndarray:
    """The HSA denoising loop over T global iterations ([TS] 2.1-2.4).

    Per iteration i: A_i from the schedule; embed the active latent rows; every
    layer on A_i with its own KV cache; head -> fresh velocities of A_i; cached
    Euler over all N; then (from ``regroup_from``) re-select the groups from
    the two cached velocities.  Returns x_T (float64 [N, C]).

    Conditioned blocks (reading of a real video DiT, see ``layer_forward``):
    ``mods[i][l]`` is layer l's [6, D] modulation at iteration i (it follows
    the timestep, so it changes with i), ``cross[l]`` layer l's text
    cross-attention; either may be None.
    """
    N, C = x0.shape
    D = weights["w_in"].shape[0]
    L = len(weights["layers"])
    check_budgets(T, budgets, counts, N)
    x = np.asarray(x0, dtype=np.float64).copy()
    g = np.asarray(g0, dtype=np.uint8).copy()
    v_hat = np.zeros((N, C))
    v_hat_prev = np.zeros((N, C))
    h = np.zeros((N, D))
    kc = [np.zeros((N, D)) for _ in range(L)]
    vc = [np.zeros((N, D)) for _ in range(L)]
    r0 = regroup_from(T, budgets)
    for i in range(T):
        mask = active_mask(g, i, T, budgets, m)
        idx = active_index(mask)
        h[idx] = embed(weights["w_in"], x[idx])
        for l in range(L):
            layer_forward(weights["layers"][l], h, idx, kc[l], vc[l], H, emulate_bf16,
                          mod=None if mods is None else mods[i][l],
                          cross=None if cross is None else cross[l])
        v_fresh = np.zeros((N, C))
        v_fresh[idx] = head(weights["w_head"], h[idx])
        x, v_hat, v_hat_prev = euler_step(x, v_hat, v_hat_prev, v_fresh, mask,
                                          sigmas[i], sigmas[i + 1])
        if regroup and r0 <= i < T - 1:
            score = l1_relative_change(v_hat_prev.astype(np.float32), v_hat.astype(np.float32))
            g = assign_groups(score, counts)
        if log is not None:
            log.append({"i": i, "idx": idx, "g": g.copy(), "x": x.copy()})
    return x


def dense_loop(weights: dict, x0: np.ndarray, T: int, sigmas: np.ndarray, H: int,
               emulate_bf16: bool = False) -> np.ndarray:
    """Uniform flow-matching sampling: every token active at every step.

    This is the full-budget baseline the method is compared against; it keeps
    no KV cache and no velocity cache.
    """
    x = np.asarray(x0, dtype=np.float64).copy()
    for i in range(T):
        h = embed(weights["w_in"], x)
        for lw in weights["layers"]:
            rb = bf16 if emulate_bf16 else (lambda t: t)
            D = h.shape[1]
            u = rb(layer_norm(h))
            qkv = u @ np.asarray(lw["w_qkv"], dtype=np.float64).T
            q, k, v = rb(qkv[:, :D]), rb(qkv[:, D:2 * D]), rb(qkv[:, 2 * D:])
            h = h + attention(q, k, v, H, emulate_bf16) @ np.asarray(lw["w_o"], dtype=np.float64).T
            u2 = rb(layer_norm(h))
            h = h + rb(gelu(u2 @ np.asarray(lw["w_1"], dtype=np.float64).T)) @ np.asarray(lw["w_2"], dtype=np.float64).T
        v = head(weights["w_head"], h)
        x = x + (float(sigmas[i + 1]) - float(sigmas[i])) * v
    return x
