"""The sampled-row block references used at full size equal the oracle's
whole-block ``layer_forward`` on small cases (active rows, fresh K/V rows and
untouched rows alike), so the full-size GPU tests compare against the pinned
block and not against a second, unchecked restatement."""

import numpy as np
import pytest

import sampled_block as SB
from oracle import hsa_oracle as O
from token_sparse_denoising_layer_b200 import synth


@pytest.mark.parametrize("N,D,H,F,a", [(40, 16, 2, 32, 17), (33, 24, 3, 40, 33), (12, 8, 1, 16, 1)])
def test_sampled_references_equal_layer_forward(N, D, H, F, a):
    w = {k: v.astype(np.float64) for k, v in synth.layer_weights(D, F, 40 + N).items()}
    x = synth.hidden_rows(N, D, 40 + N)
    ks, vs = synth.stale_kv(N, D, 40 + N)
    idx = synth.random_active_set(N, a, 40 + N)
    xr = x.astype(np.float64).copy()
    kc, vc = ks.astype(np.float64).copy(), vs.astype(np.float64).copy()
    O.layer_forward(w, xr, idx, kc, vc, H)
    rows = np.unique(np.r_[0, np.arange(a)[::3], a - 1])
    x_s, k_s, v_s = SB.block_rows(w, x, idx, ks, vs, H, rows)
    assert np.allclose(x_s, xr[idx[rows]], rtol=0, atol=1e-12)
    assert np.allclose(k_s, kc[idx[rows]], rtol=0, atol=1e-12)
    assert np.allclose(v_s, vc[idx[rows]], rtol=0, atol=1e-12)
    k2, v2 = SB.kv_rows(w, x, idx, rows)
    assert np.allclose(k2, kc[idx[rows]], rtol=0, atol=1e-12)
    assert np.allclose(v2, vc[idx[rows]], rtol=0, atol=1e-12)
    x3 = SB.block_rows_given_cache(w, x, idx, kc, vc, H, rows)
    assert np.allclose(x3, xr[idx[rows]], rtol=0, atol=1e-12)


def test_sampled_reference_sees_a_dropped_residual():
    """A block that forgot the MLP residual would differ from the reference."""
    N, D, H, F, a = 20, 8, 2, 16, 9
    w = {k: v.astype(np.float64) for k, v in synth.layer_weights(D, F, 7).items()}
    x = synth.hidden_rows(N, D, 7)
    ks, vs = synth.stale_kv(N, D, 7)
    idx = synth.random_active_set(N, a, 7)
    rows = np.arange(a)
    x_s, _, _ = SB.block_rows(w, x, idx, ks, vs, H, rows)
    tr = {}
    O.layer_forward(w, x.astype(np.float64).copy(), idx, ks.astype(np.float64).copy(),
                    vs.astype(np.float64).copy(), H, trace=tr)
    x1_only = x[idx].astype(np.float64) + tr["o"] @ w["w_o"].T
    assert not np.allclose(x_s, x1_only, atol=1e-3)
    assert np.allclose(x_s, x1_only + tr["hmid"] @ w["w_2"].T, atol=1e-12)
