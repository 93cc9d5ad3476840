"""GPU parity of the conditioned block: timestep modulation and text
cross-attention, applied to the active set only (skipped tokens incur neither,
Technical Summary: Heterogeneous Step Allocation (HSA), section 2.2 step 4).

hsa_attention_kv against the oracle's attention over an explicit key set;
hsa_layer_forward_cond against the oracle's layer_forward with ``mod`` and
``cross``, at small ragged sizes and at the 30-layer DiT's layer size on
sampled rows.  Neutral modulation must give hsa_layer_forward's result bit for
bit, zero gates must leave x untouched.
"""

import numpy as np
import pytest

from gpu_util import BF16_TOL, bf, dev, host, need_gpu, normwise, torch
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import abi, synth

pytestmark = pytest.mark.gpu

_KEYS = ("w_qkv", "w_o", "w_1", "w_2")


def _ctx(N, D, H, F):
    return abi.hsa_create(N=N, D=D, H=H, F=F, L=1, T=1, budgets=[1], counts=[N])


def _device_cross(c):
    return abi.cross_attn(bf(c["w_q"]), bf(c["w_o"]), bf(c["k_txt"]), bf(c["v_txt"]),
                          c["k_txt"].shape[0])


@pytest.mark.parametrize("n,n_kv,D,H", [
    (333, 77, 256, 2),      # one ragged key tile, ragged query tile
    (1, 1, 128, 1),         # a single key
    (2000, 512, 1536, 12),  # text-length key set at the 30-layer DiT's width
    (700, 300, 128, 2),     # head_dim 64
    (5000, 4096, 256, 2),
])
def test_attention_kv(n, n_kv, D, H):
    need_gpu()
    ctx = _ctx(max(n, n_kv), D, H, 64)
    q, k, v = synth.attention_inputs(n, n_kv, D, 12, q_scale=3.0)
    o = torch.empty((n, D), dtype=torch.bfloat16, device="cuda")
    abi.hsa_attention_kv(ctx, bf(q), n, bf(k), bf(v), n_kv, o)
    abi.hsa_sync_check(ctx)
    assert normwise(host(o), O.attention(q, k, v, H)) <= BF16_TOL


def test_attention_kv_rejects_empty_key_set():
    need_gpu()
    ctx = _ctx(256, 128, 1, 64)
    q = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_attention_kv(ctx, q, 4, q, q, 0, q)
    assert e.value.status == 3


def _run_cond(N, D, H, F, a, n_txt, use_mod, use_cross, seed):
    ctx = _ctx(N, D, H, F)
    w = synth.layer_weights(D, F, seed)
    x = synth.hidden_rows(N, D, seed)
    ks, vs = synth.stale_kv(N, D, seed)
    idx = synth.random_active_set(N, a, seed)
    mod = synth.modulation(D, seed) if use_mod else None
    cross = synth.cross_attention_weights(D, n_txt, seed) if use_cross else None
    xd, kc, vc = dev(x), bf(ks), bf(vs)
    lw = abi.layer_weights(*(bf(w[k]) for k in _KEYS))
    abi.hsa_layer_forward_cond(ctx, lw, dev(mod) if use_mod else None,
                               _device_cross(cross) if use_cross else None,
                               xd, dev(idx), a, kc, vc)
    abi.hsa_sync_check(ctx)
    return ctx, w, x, ks, vs, idx, mod, cross, xd, kc, vc


@pytest.mark.parametrize("N,D,H,F,a,n_txt,use_mod,use_cross", [
    (700, 256, 2, 512, 333, 77, True, True),
    (700, 256, 2, 512, 333, 77, True, False),
    (700, 256, 2, 512, 333, 77, False, True),
    (256, 128, 2, 512, 128, 1, True, True),
    (1500, 1536, 12, 6144, 260, 512, True, True),
])
def test_layer_forward_cond(N, D, H, F, a, n_txt, use_mod, use_cross):
    need_gpu()
    ctx, w, x, ks, vs, idx, mod, cross, xd, kc, vc = _run_cond(N, D, H, F, a, n_txt, use_mod,
                                                               use_cross, 13)
    xr = x.astype(np.float64).copy()
    kr, vr = ks.astype(np.float64).copy(), vs.astype(np.float64).copy()
    O.layer_forward(w, xr, idx, kr, vr, H, mod=mod, cross=cross)
    xg = host(xd)
    rest = np.setdiff1d(np.arange(N), idx)
    assert (xg[rest] == x[rest]).all()
    assert normwise(xg[idx] - x[idx], xr[idx] - x[idx]) <= BF16_TOL
    assert normwise(host(kc)[idx], kr[idx]) <= BF16_TOL
    assert normwise(host(vc)[idx], vr[idx]) <= BF16_TOL
    kh = host(kc)
    assert (kh[rest] == ks[rest]).all()
    ctx.close()


def test_neutral_modulation_is_the_plain_block_bitwise():
    """shift = scale = 0, gate = 1: (1 + 0) * y + 0 and 1 * acc + x are exact,
    so the conditioned block must reproduce hsa_layer_forward bit for bit."""
    need_gpu()
    N, D, H, F, a = 700, 256, 2, 512, 333
    ctx = _ctx(N, D, H, F)
    w = synth.layer_weights(D, F, 14)
    x = synth.hidden_rows(N, D, 14)
    ks, vs = synth.stale_kv(N, D, 14)
    idx = dev(synth.random_active_set(N, a, 14))
    lw = abi.layer_weights(*(bf(w[k]) for k in _KEYS))
    mod = np.zeros((6, D), np.float32)
    mod[2] = mod[5] = 1.0
    x1, k1, v1 = dev(x), bf(ks), bf(vs)
    abi.hsa_layer_forward(ctx, lw, x1, idx, a, k1, v1)
    x2, k2, v2 = dev(x), bf(ks), bf(vs)
    abi.hsa_layer_forward_cond(ctx, lw, dev(mod), None, x2, idx, a, k2, v2)
    abi.hsa_sync_check(ctx)
    assert torch.equal(x1, x2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    ctx.close()


def test_zero_gates_leave_x_untouched():
    need_gpu()
    N, D, H, F, a = 700, 256, 2, 512, 333
    ctx = _ctx(N, D, H, F)
    w = synth.layer_weights(D, F, 15)
    x = synth.hidden_rows(N, D, 15)
    ks, vs = synth.stale_kv(N, D, 15)
    idx = synth.random_active_set(N, a, 15)
    mod = synth.modulation(D, 15)
    mod[2] = mod[5] = 0.0
    lw = abi.layer_weights(*(bf(w[k]) for k in _KEYS))
    xd, kc, vc = dev(x), bf(ks), bf(vs)
    abi.hsa_layer_forward_cond(ctx, lw, dev(mod), None, xd, dev(idx), a, kc, vc)
    abi.hsa_sync_check(ctx)
    assert (host(xd) == x).all()
    # the K/V rows of the active tokens are still refreshed
    kr, vr = ks.astype(np.float64).copy(), vs.astype(np.float64).copy()
    O.layer_forward(w, x.astype(np.float64).copy(), idx, kr, vr, H, mod=mod)
    assert normwise(host(kc)[idx], kr[idx]) <= BF16_TOL
    ctx.close()


def test_cond_argument_errors():
    need_gpu()
    N, D, H, F = 256, 128, 2, 512
    ctx = _ctx(N, D, H, F)
    w = synth.layer_weights(D, F, 16)
    lw = abi.layer_weights(*(bf(w[k]) for k in _KEYS))
    x = dev(synth.hidden_rows(N, D, 16))
    kc = torch.zeros((N, D), dtype=torch.bfloat16, device="cuda")
    idx = dev(np.arange(4, dtype=np.int32))
    cross = synth.cross_attention_weights(D, 8, 16)
    xa = _device_cross(cross)
    xa.n_txt = 0
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_layer_forward_cond(ctx, lw, None, xa, x, idx, 4, kc, kc.clone())
    assert e.value.status == 3
    mod = torch.zeros(6 * D + 4, dtype=torch.float32, device="cuda")
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_layer_forward_cond(ctx, lw, mod[1:], None, x, idx, 4, kc, kc.clone())
    assert e.value.status == 1
    # a misaligned text-key pointer is refused on the host, before any launch
    k_txt = bf(cross["k_txt"])
    xa2 = _device_cross(cross)
    xa2.k_txt = k_txt.data_ptr() + 2
    with pytest.raises(abi.HsaError) as e:
        abi.hsa_layer_forward_cond(ctx, lw, None, xa2, x, idx, 4, kc, kc.clone())
    assert e.value.status == 1
    ctx.close()


def test_cond_full_size_sampled():
    """The 30-layer DiT's layer (N = 32760, D = 1536, F = 8960), 40% active,
    with modulation and 512 text tokens, on sampled active rows.  The oracle
    fills the cache with every active row's fresh K/V, then runs its block on
    the sampled rows alone: their results depend on the rest only through it."""
    need_gpu()
    N, D, H, F, a, n_txt = 32760, 1536, 12, 8960, 13104, 512
    ctx, w, x, ks, vs, idx, mod, cross, xd, kc, vc = _run_cond(N, D, H, F, a, n_txt, True, True,
                                                               17)
    u = O.layer_norm(x[idx]) * (1.0 + mod[1].astype(np.float64)) + mod[0]
    kv = O.linear(u, w["w_qkv"][D:])
    kr, vr = ks.astype(np.float64), vs.astype(np.float64)
    kr[idx] = kv[:, :D]
    vr[idx] = kv[:, D:]
    r = synth.rng(18)
    rows = np.unique(np.concatenate([[0, a - 1], r.choice(a, size=126, replace=False)]))
    sel = idx[rows]
    xr = x.astype(np.float64).copy()
    O.layer_forward(w, xr, sel, kr.copy(), vr.copy(), H, mod=mod, cross=cross)
    xg = host(xd)
    assert normwise(xg[sel] - x[sel], xr[sel] - x[sel]) <= BF16_TOL
    assert normwise(host(kc)[sel], kr[sel]) <= BF16_TOL
    skipped = np.setdiff1d(np.arange(N), idx)
    s = r.choice(skipped, size=512, replace=False)
    assert (xg[s] == x[s]).all()
    ctx.close()


def _cond_loop_setup(seed):
    from token_sparse_denoising_layer_b200.loop import HsaLoop

    spec = synth.WORKLOADS["tiny_dit"]
    sh = spec["shape"]
    counts = synth.group_counts(sh.N, spec["fractions"])
    w = synth.model_weights(sh, seed)
    layers = [tuple(bf(lw[k]) for k in _KEYS) for lw in w["layers"]]
    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, dev(w["w_in"]), dev(w["w_head"]), spec["T"],
                   spec["budgets"], counts, shift=spec["shift"])
    x0 = synth.latent(sh.N, 16, seed)
    g0 = synth.random_split(sh.N, counts, seed)
    return spec, sh, counts, w, loop, x0, g0


def test_conditioned_loop_against_oracle():
    """The tiny DiT loop with per-iteration modulation of every layer and text
    cross-attention (16 tokens) in every layer, against the float64 oracle."""
    need_gpu()
    spec, sh, counts, w, loop, x0, g0 = _cond_loop_setup(40)
    T, L = spec["T"], sh.L
    mods = [[synth.modulation(sh.D, 100 + i * L + l, spread=0.3) for l in range(L)]
            for i in range(T)]
    cross = [synth.cross_attention_weights(sh.D, 16, 200 + l) for l in range(L)]
    mods_dev = [[dev(m) for m in row] for row in mods]
    xa = [_device_cross(c) for c in cross]
    loop.reset(x0, g0)
    for i in range(T):
        loop.step(i, True, cond=abi.StepCond(mods_dev[i], xa))
    abi.hsa_sync_check(loop.ctx)
    xr = O.run_loop(w, x0, g0, T, list(spec["budgets"]), counts,
                    O.sigma_schedule(T, spec["shift"]), sh.H, mods=mods, cross=cross)
    drift = float(np.linalg.norm(host(loop.x) - xr) / np.linalg.norm(xr))
    plain = O.run_loop(w, x0, g0, T, list(spec["budgets"]), counts,
                       O.sigma_schedule(T, spec["shift"]), sh.H)
    effect = float(np.linalg.norm(plain - xr) / np.linalg.norm(xr))
    print(f"conditioned tiny-DiT loop: drift {drift:.2e} vs oracle; conditioning moves x_T by "
          f"{effect:.2e}")
    assert drift <= 2e-2 and effect > 10 * drift
    loop.close()


def test_conditioned_loop_neutral_is_the_plain_loop_bitwise():
    need_gpu()
    spec, sh, counts, w, loop, x0, g0 = _cond_loop_setup(41)
    loop.reset(x0, g0)
    loop.run(regroup=True)
    plain = host(loop.x)
    neutral = np.zeros((6, sh.D), np.float32)
    neutral[2] = neutral[5] = 1.0
    nd = dev(neutral)
    cond = abi.StepCond([nd] * sh.L, None)
    loop.reset(x0, g0)
    for i in range(spec["T"]):
        loop.step(i, True, cond=cond)
    abi.hsa_sync_check(loop.ctx)
    assert np.array_equal(host(loop.x), plain)
    loop.close()
