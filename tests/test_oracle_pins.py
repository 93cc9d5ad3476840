"""Pins for the CPU oracle: each test checks it against something other than itself.

Anchors used: hand-derived golden fixtures (tests/golden, each cited), exact
rational arithmetic, textbook double loops with ``math`` functions on tiny
inputs, closed forms, and invariants of the method as the pages state it
("Technical Summary: Heterogeneous Step Allocation (HSA) for Efficient Video
Generation", sections 2.1-2.4).  Planted-mistake tests at the end show that a
plausible slip in the oracle fails one of these pins.
"""

import math
from fractions import Fraction

import numpy as np
import pytest

from conftest import golden_rows
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import synth


# ---------------------------------------------------------------- schedule (2.1)

def _divisors(T):
    return [s for s in range(1, T + 1) if T % s == 0]


def test_schedule_equally_spaced_budget_points():
    """For every T <= 64 and every divisor budget s, a token is active at exactly
    s iterations, starting at 0, equally spaced, and covering [0, T)."""
    for T in range(1, 65):
        for s in _divisors(T):
            budgets = [T] + ([s] if s != T else [])
            k = len(budgets) - 1
            g = np.array([k], dtype=np.uint8)
            on = [i for i in range(T) if O.active_mask(g, i, T, budgets)[0]]
            assert len(on) == s
            assert on[0] == 0
            gaps = {b - a for a, b in zip(on, on[1:])} | {T - on[-1]}
            assert gaps == {T // s}


def test_schedule_golden_T40():
    rows = golden_rows("schedule_T40_budgets_40_20_10.txt")
    budgets = [40, 20, 10]
    g = np.array([0, 1, 2], dtype=np.uint8)
    assert len(rows) == 40
    for i_s, groups in rows:
        i = int(i_s)
        want = sorted(int(x) for x in groups.split(","))
        got = sorted(int(k) for k in np.flatnonzero(O.active_mask(g, i, 40, budgets)))
        assert got == want, i


def test_schedule_lay_example():
    for b, count, first in golden_rows("lay_example_T40.txt"):
        budgets = [40] if int(b) == 40 else [40, int(b)]
        g = np.array([len(budgets) - 1], dtype=np.uint8)
        on = [i for i in range(40) if O.active_mask(g, i, 40, budgets)[0]]
        assert len(on) == int(count)
        assert on[:3] == [int(x) for x in first.split(",")]


def test_active_fraction_pattern_golden():
    spec = synth.WORKLOADS["dit30_1536"]
    N = spec["shape"].N
    counts = synth.group_counts(N, spec["fractions"])
    assert counts == [13104, 9828, 9828]
    classes = {"i%4==0": lambda i: i % 4 == 0, "i%4==2": lambda i: i % 4 == 2,
               "i%2==1": lambda i: i % 2 == 1}
    g = synth.random_split(N, counts, 0)
    for cls, n_i, tokens in golden_rows("pattern_fractions_dit30.txt"):
        its = [i for i in range(40) if classes[cls](i)]
        assert len(its) == int(n_i)
        for i in its:
            assert O.n_active(i, 40, spec["budgets"], counts) == int(tokens)
            assert int(O.active_mask(g, i, 40, spec["budgets"]).sum()) == int(tokens)
    mean = np.mean([O.n_active(i, 40, spec["budgets"], counts) for i in range(40)]) / N
    assert abs(mean - 0.625) < 1e-12


def test_baseline_group_always_active_and_index_ascending():
    r = np.random.default_rng(3)
    g = r.integers(0, 3, 500).astype(np.uint8)
    for i in range(40):
        mask = O.active_mask(g, i, 40, [40, 20, 10])
        assert mask[g == 0].all()
        idx = O.active_index(mask)
        assert idx.dtype == np.int32
        assert np.all(np.diff(idx) > 0)
        assert set(idx.tolist()) == {n for n in range(500) if mask[n]}


def test_phase_window_full_passes():
    g = np.array([0, 1, 2] * 10, dtype=np.uint8)
    T, m = 40, 3
    for i in range(T):
        mask = O.active_mask(g, i, T, [40, 20, 10], m)
        if i < m or i >= T - m:
            assert mask.all()
        else:
            assert (mask == O.active_mask(g, i, T, [40, 20, 10], 0)).all()


def test_budget_validation():
    O.check_budgets(40, [40, 20, 10], [4, 3, 3], 10)
    with pytest.raises(ValueError):
        O.check_budgets(40, [40, 15], None)      # 15 does not divide 40
    with pytest.raises(ValueError):
        O.check_budgets(40, [20, 10], None)      # s_1 != T
    with pytest.raises(ValueError):
        O.check_budgets(40, [40, 20], [5, 4], 10)


# ---------------------------------------------------------------- selection (2.1)

def _score_exact(vp, vc, eps):
    """L1 relative change in exact rational arithmetic."""
    num = sum(abs(Fraction(float(b)) - Fraction(float(a))) for a, b in zip(vp, vc))
    den = sum(abs(Fraction(float(a))) for a in vp) + Fraction(eps)
    return num / den


def test_score_against_exact_rationals():
    r = np.random.default_rng(5)
    vp = r.standard_normal((40, 16)).astype(np.float32)
    vc = r.standard_normal((40, 16)).astype(np.float32)
    vc[:10] = vp[:10] + np.float32(0.01) * r.standard_normal((10, 16)).astype(np.float32)
    got = O.l1_relative_change(vp, vc)
    got64 = O.l1_relative_change_f64(vp, vc)
    for n in range(40):
        exact = float(_score_exact(vp[n], vc[n], O.SCORE_EPS))
        # 16 float32 additions per sum, one subtraction, one division
        assert abs(got[n] - exact) <= 40 * 2.0 ** -24 * exact + 1e-30
        assert abs(got64[n] - exact) <= 1e-13 * exact + 1e-300


def test_score_closed_forms():
    vp = np.tile(np.array([1, -2, 0.5, 4] * 4, dtype=np.float32), (3, 1))
    S = float(np.abs(vp[0]).sum())
    vc = np.stack([vp[0], vp[0] * np.float32(1.5), -vp[0]])
    r = O.l1_relative_change(vp, vc)
    assert r[0] == 0.0 and not np.signbit(r[0])
    assert abs(r[1] - 0.5 * S / (S + 1e-6)) < 1e-7
    assert abs(r[2] - 2.0 * S / (S + 1e-6)) < 1e-7


def test_selection_brute_force_sorted_tuples():
    for seed in range(6):
        N = 37 + seed
        s = synth.score_buffer(N, seed, n_tie_values=4 if seed % 2 else 0)
        counts = synth.group_counts(N, (0.4, 0.3, 0.3))
        g = O.assign_groups(s, counts)
        ranked = sorted(range(N), key=lambda n: (-float(s[n]), n))
        want = np.empty(N, dtype=np.uint8)
        bounds = np.cumsum([0] + counts)
        for k in range(3):
            for n in ranked[bounds[k]:bounds[k + 1]]:
                want[n] = k
        assert (g == want).all()
        assert [int((g == k).sum()) for k in range(3)] == counts


def test_selection_ties_go_to_lower_index():
    s = np.array([1.0, 2.0, 2.0, 2.0, 0.5, 2.0], dtype=np.float32)
    g = O.assign_groups(s, [2, 2, 2])
    # ranking: 1, 2, 3, 5 (all 2.0, by index), then 0, then 4
    assert g.tolist() == [2, 0, 0, 1, 2, 1]


def test_selection_low_change_region_lands_in_slowest_group():
    """30% of tokens change by 1% -> exactly those tokens form the 30% slow group."""
    for contiguous in (False, True):
        N = 3000
        vp, vc, low = synth.velocity_pair(N, 16, 1, contiguous=contiguous)
        counts = synth.group_counts(N, (0.4, 0.3, 0.3))
        g = O.assign_groups(O.l1_relative_change(vp, vc), counts)
        assert (g[low] == 2).all()
        assert ((g == 2) == low).all()
        assert int((g == 0).sum()) == counts[0]


def test_selection_rejects_nan():
    with pytest.raises(ValueError):
        O.assign_groups(np.array([0.1, np.nan], dtype=np.float32), [1, 1])


# ---------------------------------------------------------------- layer pieces

def _ln_loops(row, eps=1e-5):
    D = len(row)
    mu = math.fsum(row) / D
    var = math.fsum((v - mu) ** 2 for v in row) / D
    return [(v - mu) / math.sqrt(var + eps) for v in row]


def test_layer_norm_textbook_and_invariants():
    r = np.random.default_rng(7)
    x = r.standard_normal((5, 24)) * 3 + 2
    y = O.layer_norm(x)
    for i in range(5):
        assert np.allclose(y[i], _ln_loops(list(x[i])), atol=1e-12)
    assert np.allclose(y.mean(axis=1), 0, atol=1e-12)
    assert np.allclose(O.layer_norm(np.full((2, 8), 3.0)), 0)
    assert np.allclose(O.layer_norm(7.0 * x + 1.0), y, atol=1e-5)


def test_gelu_known_values():
    assert O.gelu(np.array([0.0]))[0] == 0.0
    # Phi(1) = 0.8413447460685429 (standard normal table)
    assert abs(O.gelu(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15
    x = np.linspace(-4, 4, 33)
    assert np.allclose(O.gelu(x) - O.gelu(-x), x, atol=1e-14)   # x*Phi(x) - (-x)Phi(-x) = x
    assert abs(O.gelu(np.array([10.0]))[0] - 10.0) < 1e-12


def _attn_loops(q, K, V, H):
    a, D = len(q), len(q[0])
    d = D // H
    out = [[0.0] * D for _ in range(a)]
    for i in range(a):
        for h in range(H):
            s = [sum(q[i][h * d + t] * K[j][h * d + t] for t in range(d)) / math.sqrt(d)
                 for j in range(len(K))]
            mx = max(s)
            e = [math.exp(v - mx) for v in s]
            z = math.fsum(e)
            for t in range(d):
                out[i][h * d + t] = math.fsum(e[j] * V[j][h * d + t] for j in range(len(K))) / z
    return out


def test_attention_textbook_loops():
    r = np.random.default_rng(9)
    q = r.standard_normal((3, 8)) * 2
    K = r.standard_normal((7, 8))
    V = r.standard_normal((7, 8))
    got = O.attention(q, K, V, H=2)
    want = np.array(_attn_loops(q.tolist(), K.tolist(), V.tolist(), 2))
    assert np.allclose(got, want, atol=1e-12)


def test_attention_identical_keys_give_mean_of_values():
    r = np.random.default_rng(10)
    K = np.tile(r.standard_normal((1, 16)), (9, 1))
    V = r.standard_normal((9, 16))
    q = r.standard_normal((4, 16)) * 5
    got = O.attention(q, K, V, H=2)
    assert np.allclose(got, np.tile(V.mean(axis=0), (4, 1)), atol=1e-12)


def test_attention_peaked_query_selects_one_value_row():
    r = np.random.default_rng(11)
    K = np.eye(8) * 50.0                      # one head, d = 8, orthogonal keys
    V = r.standard_normal((8, 8))
    q = np.eye(8)[[3, 5]] * 50.0
    got = O.attention(q, K, V, H=1)
    assert np.allclose(got, V[[3, 5]], atol=1e-9)


def test_attention_key_permutation_invariance():
    r = np.random.default_rng(12)
    q, K, V = r.standard_normal((3, 16)), r.standard_normal((11, 16)), r.standard_normal((11, 16))
    p = r.permutation(11)
    assert np.allclose(O.attention(q, K, V, 2), O.attention(q, K[p], V[p], 2), atol=1e-12)


def _block_loops(w, x, H):
    """A textbook pre-LN transformer block on all rows, written with loops."""
    D = len(x[0])
    wq = w["w_qkv"]
    u = [_ln_loops(row) for row in x]
    lin = lambda W, v: [math.fsum(W[o][t] * v[t] for t in range(len(v))) for o in range(len(W))]
    qkv = [lin(wq, row) for row in u]
    q = [row[:D] for row in qkv]
    k = [row[D:2 * D] for row in qkv]
    v = [row[2 * D:] for row in qkv]
    att = _attn_loops(q, k, v, H)
    x1 = [[a + b for a, b in zip(xr, lin(w["w_o"], ar))] for xr, ar in zip(x, att)]
    u2 = [_ln_loops(row) for row in x1]
    hid = [[0.5 * t * (1 + math.erf(t / math.sqrt(2))) for t in lin(w["w_1"], row)] for row in u2]
    return [[a + b for a, b in zip(xr, lin(w["w_2"], hr))] for xr, hr in zip(x1, hid)]


def test_layer_all_active_equals_textbook_block():
    N, D, H, F = 6, 8, 2, 16
    w = {k: v.astype(np.float64) for k, v in synth.layer_weights(D, F, 3).items()}
    x = synth.hidden_rows(N, D, 3).astype(np.float64)
    want = np.array(_block_loops(w, x.tolist(), H))
    kc, vc = np.zeros((N, D)), np.zeros((N, D))
    xx = x.copy()
    O.layer_forward(w, xx, np.arange(N, dtype=np.int32), kc, vc, H)
    assert np.allclose(xx, want, atol=1e-10)


def test_layer_sparse_rows_match_textbook_with_stale_cache():
    """Active rows see fresh K/V for A_i and stale K/V for the rest; skipped rows
    of x and of the cache are untouched."""
    N, D, H, F = 9, 8, 2, 16
    w = {k: v.astype(np.float64) for k, v in synth.layer_weights(D, F, 4).items()}
    x = synth.hidden_rows(N, D, 4).astype(np.float64)
    ks, vs = synth.stale_kv(N, D, 4)
    idx = np.array([1, 4, 5, 8], dtype=np.int32)
    kc, vc = ks.astype(np.float64).copy(), vs.astype(np.float64).copy()
    xx = x.copy()
    O.layer_forward(w, xx, idx, kc, vc, H)
    skipped = np.setdiff1d(np.arange(N), idx)
    assert (xx[skipped] == x[skipped]).all()
    assert (kc[skipped] == ks[skipped]).all() and (vc[skipped] == vs[skipped]).all()
    # rebuild the expectation with loops: fresh k/v rows for idx, stale elsewhere
    lin = lambda W, v: [math.fsum(W[o][t] * v[t] for t in range(len(v))) for o in range(len(W))]
    K = ks.astype(np.float64).tolist()
    V = vs.astype(np.float64).tolist()
    qs = []
    for n in idx:
        qkv = lin(w["w_qkv"].tolist(), _ln_loops(list(x[n])))
        qs.append(qkv[:D])
        K[n], V[n] = qkv[D:2 * D], qkv[2 * D:]
    att = _attn_loops(qs, K, V, H)
    for r_, n in enumerate(idx):
        x1 = [a + b for a, b in zip(x[n], lin(w["w_o"].tolist(), att[r_]))]
        hid = [0.5 * t * (1 + math.erf(t / math.sqrt(2))) for t in lin(w["w_1"].tolist(), _ln_loops(x1))]
        x2 = [a + b for a, b in zip(x1, lin(w["w_2"].tolist(), hid))]
        assert np.allclose(xx[n], x2, atol=1e-10)


def test_refreshed_cache_gives_dense_attention():
    """Once every token has been active, attention against the cache is dense attention."""
    N, D, H, F = 10, 8, 2, 16
    w = {k: v.astype(np.float64) for k, v in synth.layer_weights(D, F, 5).items()}
    x = synth.hidden_rows(N, D, 5).astype(np.float64)
    kc, vc = np.zeros((N, D)), np.zeros((N, D))
    tr = {}
    O.layer_forward(w, x.copy(), np.arange(N, dtype=np.int32), kc, vc, H, trace=tr)
    u = O.layer_norm(x)
    qkv = u @ w["w_qkv"].T
    dense = O.attention(qkv[:, :D], qkv[:, D:2 * D], qkv[:, 2 * D:], H)
    assert np.allclose(tr["o"], dense, atol=1e-12)
    # a later sparse step: rows 0..4 refreshed, queries of rows 0..4 only
    tr2 = {}
    x2 = x.copy()
    O.layer_forward(w, x2, np.arange(5, dtype=np.int32), kc, vc, H, trace=tr2)
    assert np.allclose(tr2["o"], dense[:5], atol=1e-12)


def test_conditioning_neutral_modulation_is_the_plain_block():
    """shift = scale = 0 and gate = 1 leave the block unchanged, bit for bit."""
    N, D, H, F = 9, 8, 2, 16
    w = {k: v.astype(np.float64) for k, v in synth.layer_weights(D, F, 8).items()}
    x = synth.hidden_rows(N, D, 8).astype(np.float64)
    idx = np.array([0, 3, 4, 8], dtype=np.int32)
    m = np.zeros((6, D))
    m[2] = m[5] = 1.0
    a, b = x.copy(), x.copy()
    O.layer_forward(w, a, idx, np.zeros((N, D)), np.zeros((N, D)), H)
    O.layer_forward(w, b, idx, np.zeros((N, D)), np.zeros((N, D)), H, mod=m)
    assert (a == b).all()


def test_conditioning_zero_gates_remove_their_branch():
    """gate_a = gate_m = 0: the block only updates the caches; x is unchanged.
    gate_m = 0 alone: x gets exactly the (modulated) attention branch."""
    N, D, H, F = 9, 8, 2, 16
    w = {k: v.astype(np.float64) for k, v in synth.layer_weights(D, F, 9).items()}
    x = synth.hidden_rows(N, D, 9).astype(np.float64)
    idx = np.array([1, 2, 7], dtype=np.int32)
    m = synth.modulation(D, 9).astype(np.float64)
    m[2] = 0.0
    m[5] = 0.0
    xx = x.copy()
    O.layer_forward(w, xx, idx, np.zeros((N, D)), np.zeros((N, D)), H, mod=m)
    assert (xx == x).all()
    m2 = synth.modulation(D, 9).astype(np.float64)
    m2[5] = 0.0
    xx = x.copy()
    kc, vc = np.zeros((N, D)), np.zeros((N, D))
    tr = {}
    O.layer_forward(w, xx, idx, kc, vc, H, mod=m2, trace=tr)
    want = x[idx] + m2[2] * (tr["o"] @ w["w_o"].T)
    assert np.allclose(xx[idx], want, atol=1e-12)
    # the modulated LN input: per-channel affine map of the normalised rows
    assert np.allclose(tr["u"], O.layer_norm(x[idx]) * (1 + m2[1]) + m2[0], atol=1e-12)


def test_cross_attention_textbook_and_closed_form():
    """Cross-attention of the active queries against the text tokens: equal to a
    textbook loop computation, and with identical text keys to the mean of the
    text values."""
    N, D, H, F, T = 6, 8, 2, 16, 5
    w = {k: v.astype(np.float64) for k, v in synth.layer_weights(D, F, 10).items()}
    c = {k: v.astype(np.float64) for k, v in synth.cross_attention_weights(D, T, 10).items()}
    x = synth.hidden_rows(N, D, 10).astype(np.float64)
    idx = np.array([0, 2, 5], dtype=np.int32)
    kc, vc = np.zeros((N, D)), np.zeros((N, D))
    tr = {}
    xx = x.copy()
    O.layer_forward(w, xx, idx, kc, vc, H, trace=tr, cross=c)
    # textbook: rebuild x after self-attention, then the cross branch with loops
    x1 = x[idx] + tr["o"] @ w["w_o"].T
    lin = lambda W, v: [math.fsum(W[o][t] * v[t] for t in range(len(v))) for o in range(len(W))]
    qc = [lin(c["w_q"].tolist(), _ln_loops(list(r))) for r in x1]
    oc = _attn_loops(qc, c["k_txt"].tolist(), c["v_txt"].tolist(), H)
    assert np.allclose(tr["oc"], np.array(oc), atol=1e-12)
    # identical keys: every query sees the mean of the text values
    c2 = dict(c)
    c2["k_txt"] = np.tile(c["k_txt"][:1], (T, 1))
    tr2 = {}
    O.layer_forward(w, x.copy(), idx, np.zeros((N, D)), np.zeros((N, D)), H, trace=tr2, cross=c2)
    assert np.allclose(tr2["oc"], np.tile(c["v_txt"].mean(axis=0), (len(idx), 1)), atol=1e-12)


# ---------------------------------------------------------------- embed and velocity head

def _lin_loops(W, v):
    return [math.fsum(W[o][t] * v[t] for t in range(len(v))) for o in range(len(W))]


def test_embed_textbook_loops_and_one_hot_rows():
    """Patch embed, latent rows [a, C] -> hidden rows [a, D] with w_in [D, C]:
    hidden value o of a row is the dot product of the row with w_in's row o.
    Checked with loops, once with D = C = 16 (where a transposed w_in keeps the
    right shape), and on one-hot latent rows, which pick out one column of w_in."""
    r = np.random.default_rng(30)
    for D in (16, 8):
        w_in = r.standard_normal((D, 16))
        xl = r.standard_normal((5, 16)) * 2.0
        got = O.embed(w_in, xl)
        want = np.array([_lin_loops(w_in.tolist(), row) for row in xl.tolist()])
        assert got.shape == (5, D)
        assert np.allclose(got, want, atol=1e-12)
    w_in = r.standard_normal((16, 16))
    onehot = np.eye(16)[[0, 5, 15]]
    assert np.array_equal(O.embed(w_in, onehot), w_in[:, [0, 5, 15]].T)


def test_head_textbook_loops_and_closed_forms():
    """Velocity head, hidden rows [a, D] -> velocities [a, C] with w_head [C, D]:
    the final LayerNorm of the row (no affine, eps 1e-5), then the linear map.
    Checked with loops (D = C = 16, so a transposed w_head keeps the shape); a
    constant row normalises to zero and so predicts zero velocity; a positive
    affine change of a row leaves the prediction as it was; a row that already
    has zero mean and unit variance is only divided by sqrt(1 + eps)."""
    r = np.random.default_rng(31)
    for D in (16, 24):
        w_head = r.standard_normal((16, D))
        h = r.standard_normal((5, D)) * 3.0 + 1.5
        got = O.head(w_head, h)
        want = np.array([_lin_loops(w_head.tolist(), _ln_loops(row)) for row in h.tolist()])
        assert got.shape == (5, 16)
        assert np.allclose(got, want, atol=1e-11)
    w_head = r.standard_normal((16, 24))
    assert np.allclose(O.head(w_head, np.full((3, 24), 4.25)), 0.0, atol=1e-12)
    h = r.standard_normal((4, 24))
    assert np.allclose(O.head(w_head, 5.0 * h - 2.0), O.head(w_head, h), atol=1e-5)
    z = np.array([[1.0, -1.0] * 12])                    # mean 0, variance 1
    assert np.allclose(O.head(w_head, z), (z @ w_head.T) / math.sqrt(1.0 + 1e-5), atol=1e-13)


# ---------------------------------------------------------------- cached Euler (2.3)

def test_euler_telescoping_closed_form():
    T = 40
    sig = O.sigma_schedule(T, shift=5.0)
    r = np.random.default_rng(13)
    x0 = r.standard_normal((50, 16))
    v = r.standard_normal((50, 16))
    x, vh, vp = x0, v.copy(), np.zeros_like(v)
    mask = np.zeros(50, dtype=bool)
    for i in range(T):
        x, vh, vp = O.euler_step(x, vh, vp, np.zeros_like(v), mask, sig[i], sig[i + 1])
    assert np.allclose(x, x0 + v * (float(sig[T]) - float(sig[0])), atol=1e-12)
    assert (vh == v).all()


def test_euler_fresh_vs_cached_selection():
    r = np.random.default_rng(14)
    x, vh, vp, vf = (r.standard_normal((8, 16)) for _ in range(4))
    mask = np.array([1, 0, 1, 1, 0, 0, 1, 0], dtype=bool)
    nx, nh, npv = O.euler_step(x, vh, vp, vf, mask, 0.75, 0.5)
    assert (nh[mask] == vf[mask]).all() and (nh[~mask] == vh[~mask]).all()
    assert (npv[mask] == vh[mask]).all() and (npv[~mask] == vp[~mask]).all()
    assert np.allclose(nx, x - 0.25 * nh, atol=1e-15)


def test_euler_f32_matches_f64_within_rounding():
    r = np.random.default_rng(15)
    x, vh, vp, vf = (r.standard_normal((64, 16)).astype(np.float32) for _ in range(4))
    mask = r.random(64) < 0.5
    a = O.euler_step(x, vh, vp, vf, mask, np.float32(0.8), np.float32(0.77))
    b = O.euler_step_f32(x, vh, vp, vf, mask, np.float32(0.8), np.float32(0.77))
    assert np.allclose(a[0], b[0], rtol=0, atol=4e-7 * np.abs(a[0]).max())
    assert (a[1] == b[1]).all() and (a[2] == b[2]).all()


def test_sigma_shift_scales_the_odds():
    """The flow-matching timestep shift by a factor s multiplies the odds of
    every interior noise level by s: sigma' / (1 - sigma') = s sigma / (1 - sigma)
    with sigma = 1 - j/T (exact rationals; the table is float32).  A shift by
    1/s instead of s, or a shift of 1 - sigma, breaks it."""
    T = 40
    for shift in (5.0, 3.0):
        tab = O.sigma_schedule(T, shift)
        for j in range(1, T):
            sig = Fraction(T - j, T)
            odds = Fraction(int(shift)) * sig / (1 - sig)
            want = odds / (1 + odds)
            assert abs(Fraction(float(tab[j])) - want) <= Fraction(1, 2 ** 23), (shift, j)


def test_sigma_schedule_endpoints_and_monotone():
    for shift in (1.0, 5.0):
        s = O.sigma_schedule(40, shift)
        assert s[0] == 1.0 and s[-1] == 0.0
        assert np.all(np.diff(s) < 0)
    assert np.allclose(O.sigma_schedule(8, 1.0), 1 - np.arange(9) / 8)


# ---------------------------------------------------------------- the loop

def _tiny_model(L=1, N=24, D=16, H=2, F=32, seed=0):
    shape = synth.ModelShape(N=N, C=16, D=D, H=H, F=F, L=L)
    w = synth.model_weights(shape, seed)
    return shape, w


def test_all_active_loop_equals_dense_loop_bitwise():
    """Every s_k = T: the HSA loop is uniform flow matching, bit for bit."""
    shape, w = _tiny_model(L=2)
    x0 = synth.latent(shape.N, 16, 0)
    T = 4
    sig = O.sigma_schedule(T, 1.0)
    g0 = np.zeros(shape.N, dtype=np.uint8)
    a = O.run_loop(w, x0, g0, T, [T], [shape.N], sig, shape.H)
    b = O.dense_loop(w, x0, T, sig, shape.H)
    assert (a == b).all()


def test_loop_skipped_tokens_follow_cached_velocity():
    """A token of the slowest group moves on a straight line with the velocity of
    its last active step until it is active again (cached Euler, 2.3)."""
    shape, w = _tiny_model(L=1)
    x0 = synth.latent(shape.N, 16, 1).astype(np.float64)
    T, budgets, counts = 8, [8, 4, 2], [8, 8, 8]
    sig = O.sigma_schedule(T, 1.0).astype(np.float64)
    g0 = synth.random_split(shape.N, counts, 1)
    log = []
    O.run_loop(w, x0, g0, T, budgets, counts, sig.astype(np.float32), shape.H,
               regroup=False, log=log)
    xs = [x0] + [lg["x"] for lg in log]
    slow = g0 == 2
    for lg in log:
        on = np.zeros(shape.N, dtype=bool)
        on[lg["idx"]] = True
        assert on[slow].all() if lg["i"] % 4 == 0 else not on[slow].any()
        assert (lg["g"] == g0).all()
    v0 = (xs[1] - xs[0]) / (sig[1] - sig[0])
    v4 = (xs[4] - xs[0]) / (sig[4] - sig[0])
    assert np.allclose(v4[slow], v0[slow], atol=1e-9)
    assert not np.allclose(v4[~slow], v0[~slow], atol=1e-3)


def test_loop_regroup_keeps_counts():
    shape, w = _tiny_model(L=1)
    x0 = synth.latent(shape.N, 16, 2)
    T, budgets, counts = 8, [8, 4], [12, 12]
    log = []
    O.run_loop(w, x0, synth.random_split(shape.N, counts, 2), T, budgets, counts,
               O.sigma_schedule(T, 1.0), shape.H, log=log)
    for lg in log:
        assert [int((lg["g"] == k).sum()) for k in range(2)] == counts
    assert O.regroup_from(T, budgets) == 2


# ---------------------------------------------------------------- planted mistakes

def test_planted_mistakes_are_caught(monkeypatch):
    """A wrong sign in the Euler step, values paired with the wrong keys, a
    dropped LN eps, a head without its final LayerNorm or with w_head transposed,
    and an embed with w_in transposed or its output scaled each break one of the
    pins above."""
    orig_euler = O.euler_step

    def bad_euler(x, vh, vp, vf, mask, si, sn):
        nx, nh, npv = orig_euler(x, vh, vp, vf, mask, si, sn)
        return np.asarray(x) - (float(sn) - float(si)) * nh, nh, npv

    monkeypatch.setattr(O, "euler_step", bad_euler)
    with pytest.raises(AssertionError):
        test_euler_telescoping_closed_form()
    monkeypatch.setattr(O, "euler_step", orig_euler)

    orig_ln = O.layer_norm
    monkeypatch.setattr(O, "layer_norm", lambda x, eps=0.0: orig_ln(x, 1e-1))
    with pytest.raises(AssertionError):
        test_layer_all_active_equals_textbook_block()
    monkeypatch.setattr(O, "layer_norm", orig_ln)

    orig_att = O.attention

    def bad_att(q, K, V, H, emulate_bf16=False):
        return orig_att(q, K, V[::-1], H, emulate_bf16)   # values paired with the wrong keys

    monkeypatch.setattr(O, "attention", bad_att)
    with pytest.raises(AssertionError):
        test_attention_textbook_loops()
    monkeypatch.setattr(O, "attention", orig_att)

    orig_head = O.head
    monkeypatch.setattr(O, "head", lambda w_head, h: np.asarray(h) @ np.asarray(w_head).T)
    with pytest.raises(AssertionError):                  # final LayerNorm dropped
        test_head_textbook_loops_and_closed_forms()
    monkeypatch.setattr(O, "head", lambda w_head, h: orig_head(np.asarray(w_head).T, h)
                        if np.asarray(w_head).shape[0] == np.asarray(w_head).shape[1]
                        else orig_head(w_head, h))
    with pytest.raises(AssertionError):                  # w_head transposed
        test_head_textbook_loops_and_closed_forms()
    monkeypatch.setattr(O, "head", orig_head)

    orig_embed = O.embed
    monkeypatch.setattr(O, "embed", lambda w_in, xl: orig_embed(np.asarray(w_in).T, xl)
                        if np.asarray(w_in).shape[0] == np.asarray(w_in).shape[1]
                        else orig_embed(w_in, xl))
    with pytest.raises(AssertionError):                  # w_in transposed
        test_embed_textbook_loops_and_one_hot_rows()
    monkeypatch.setattr(O, "embed", lambda w_in, xl: 2.0 * orig_embed(w_in, xl))
    with pytest.raises(AssertionError):                  # output scaled
        test_embed_textbook_loops_and_one_hot_rows()
    monkeypatch.setattr(O, "embed", orig_embed)


def _cond_model(seed):
    sh = synth.ModelShape(N=24, C=16, D=8, H=2, F=16, L=2)
    w = synth.model_weights(sh, seed)
    w = {"w_in": w["w_in"].astype(np.float64), "w_head": w["w_head"].astype(np.float64),
         "layers": [{k: v.astype(np.float64) for k, v in lw.items()} for lw in w["layers"]]}
    return sh, w


def test_conditioned_loop_neutral_is_the_plain_loop():
    """Neutral modulation at every iteration and cross-attention whose output
    projection is zero leave the whole loop bit for bit as the plain loop."""
    sh, w = _cond_model(21)
    T, budgets, counts = 8, [8, 4, 2], [8, 8, 8]
    x0 = synth.latent(sh.N, 16, 21)
    g0 = synth.random_split(sh.N, counts, 21)
    sig = O.sigma_schedule(T, 1.0)
    neutral = np.zeros((6, sh.D))
    neutral[2] = neutral[5] = 1.0
    mods = [[neutral] * sh.L for _ in range(T)]
    cross = []
    for l in range(sh.L):
        c = synth.cross_attention_weights(sh.D, 5, 21 + l)
        c = {k: v.astype(np.float64) for k, v in c.items()}
        c["w_o"] = np.zeros_like(c["w_o"])
        cross.append(c)
    plain = O.run_loop(w, x0, g0, T, budgets, counts, sig, sh.H)
    cond = O.run_loop(w, x0, g0, T, budgets, counts, sig, sh.H, mods=mods, cross=cross)
    assert (plain == cond).all()


def test_conditioned_loop_uses_each_iterations_modulation_at_that_iteration():
    """Modulation that departs from neutral only at the last iteration leaves
    every earlier iterate unchanged and changes the last one."""
    sh, w = _cond_model(22)
    T, budgets, counts = 8, [8, 4], [12, 12]
    x0 = synth.latent(sh.N, 16, 22)
    g0 = synth.random_split(sh.N, counts, 22)
    sig = O.sigma_schedule(T, 1.0)
    neutral = np.zeros((6, sh.D))
    neutral[2] = neutral[5] = 1.0
    mods = [[neutral] * sh.L for _ in range(T)]
    mods[T - 1] = [synth.modulation(sh.D, 22 + l).astype(np.float64) for l in range(sh.L)]
    la, lb = [], []
    O.run_loop(w, x0, g0, T, budgets, counts, sig, sh.H, log=la)
    O.run_loop(w, x0, g0, T, budgets, counts, sig, sh.H, log=lb, mods=mods)
    for i in range(T - 1):
        assert (la[i]["x"] == lb[i]["x"]).all()
    assert not (la[T - 1]["x"] == lb[T - 1]["x"]).all()
