"""Oracle block outputs on sampled active rows, for parity at full size.

At the workloads' full sizes the oracle cannot run a whole block, so the GPU
block ("Technical Summary: Heterogeneous Step Allocation (HSA) for Efficient
Video Generation", section 2.2: QKV of A_i, fresh K/V rows into the cache,
attention of A_i against all N rows, out-projection and MLP on A_i) is checked
on a sample of its active rows.  Each function here is the oracle's
``layer_forward`` restricted to those rows, built from the oracle's pieces;
tests/test_sampled_block.py checks every one of them against
``layer_forward`` itself on small cases.
"""

import numpy as np

from oracle import hsa_oracle as O


def kv_rows(w, x, idx, rows):
    """Fresh K and V (float64) of the active rows idx[rows]."""
    D = x.shape[1]
    kv = O.linear(O.layer_norm(x[idx[rows]]), w["w_qkv"][D:])
    return kv[:, :D], kv[:, D:]


def full_cache(w, x, idx, ks, vs):
    """The cache after the block's write: every active row's fresh K and V
    (float64) over the stale rows ks, vs."""
    D = x.shape[1]
    kv = O.linear(O.layer_norm(x[idx]), w["w_qkv"][D:])
    kc = ks.astype(np.float64)
    vc = vs.astype(np.float64)
    kc[idx] = kv[:, :D]
    vc[idx] = kv[:, D:]
    return kc, vc


def block_rows_given_cache(w, x, idx, kc, vc, H, rows):
    """Block output x rows idx[rows], given the cache as it stands after the
    block's write (every active row fresh).  Attention runs one head at a time,
    so a cache of any size is read in float64 one head's columns at a time."""
    D = x.shape[1]
    d = D // H
    xa = x[idx[rows]].astype(np.float64)
    q = O.linear(O.layer_norm(xa), w["w_qkv"][:D])
    o = np.empty_like(q)
    for h in range(H):
        sl = slice(h * d, (h + 1) * d)
        o[:, sl] = O.attention(q[:, sl], kc[:, sl], vc[:, sl], 1)
    x1 = xa + O.linear(o, w["w_o"])
    return x1 + O.linear(O.gelu(O.linear(O.layer_norm(x1), w["w_1"])), w["w_2"])


def block_rows(w, x, idx, ks, vs, H, rows):
    """Block outputs for the active rows idx[rows], the cache rebuilt by the
    oracle from every active row: (x rows, K rows, V rows)."""
    kc, vc = full_cache(w, x, idx, ks, vs)
    return block_rows_given_cache(w, x, idx, kc, vc, H, rows), kc[idx[rows]], vc[idx[rows]]
