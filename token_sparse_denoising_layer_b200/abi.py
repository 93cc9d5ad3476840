"""Thin ctypes binding of libhsa.so: the same names as the C ABI in include/hsa.h.

Only argument marshalling happens here.  Tensors are passed by device
address (``tensor.data_ptr()``); every step of the HSA path runs in the
library's CUDA kernels.  There is no fallback: if libhsa.so is missing, or a
call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libhsa.so")

# Every symbol the header declares, in header order.
SYMBOLS = [
    "hsa_create", "hsa_destroy", "hsa_last_error", "hsa_set_stream", "hsa_sync_check",
    "hsa_selftest_timeout", "hsa_kernel_launches", "hsa_time_kernels", "hsa_kernel_times", "hsa_n_active", "hsa_schedule", "hsa_score", "hsa_select_from_score",
    "hsa_select_groups", "hsa_ln_gather", "hsa_qkv_project", "hsa_qkv_project_peers", "hsa_linear", "hsa_kv_scatter", "hsa_kv_scatter_packed",
    "hsa_attention", "hsa_attention_kv", "hsa_out_proj_residual", "hsa_mlp_residual",
    "hsa_ln_gather_mod", "hsa_out_proj_residual_gated", "hsa_mlp_residual_mod",
    "hsa_layer_forward", "hsa_layer_forward_cond", "hsa_embed", "hsa_head", "hsa_euler_step", "hsa_euler_step_score", "hsa_step", "hsa_step_cond",
    "hsa_select_groups_static",
]

STATUS = {0: "HSA_OK", 1: "HSA_ERR_INVALID_ARG", 2: "HSA_ERR_BUDGET", 3: "HSA_ERR_SHAPE",
          4: "HSA_ERR_CUDA", 5: "HSA_ERR_OOM", 6: "HSA_ERR_TIMEOUT", 7: "HSA_ERR_DEVICE_CHECK",
          8: "HSA_ERR_SCRATCH_LIMIT"}

SELECT_STATIC_MAX_N = 131072  # HSA_SELECT_STATIC_MAX_N in include/hsa.h


class HsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class hsa_model_cfg(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("C", ctypes.c_int), ("D", ctypes.c_int),
                ("H", ctypes.c_int), ("F", ctypes.c_int), ("L", ctypes.c_int)]


class hsa_layer_weights(ctypes.Structure):
    _fields_ = [("w_qkv", ctypes.c_void_p), ("w_o", ctypes.c_void_p),
                ("w_1", ctypes.c_void_p), ("w_2", ctypes.c_void_p)]


class hsa_cross_attn(ctypes.Structure):
    _fields_ = [("w_q", ctypes.c_void_p), ("w_o", ctypes.c_void_p), ("k_txt", ctypes.c_void_p),
                ("v_txt", ctypes.c_void_p), ("n_txt", ctypes.c_int)]


class hsa_cond(ctypes.Structure):
    _fields_ = [("mod", ctypes.POINTER(ctypes.c_void_p)), ("xa", ctypes.POINTER(hsa_cross_attn))]


class hsa_model_weights(ctypes.Structure):
    _fields_ = [("w_in", ctypes.c_void_p), ("w_head", ctypes.c_void_p),
                ("layers", ctypes.POINTER(hsa_layer_weights))]


class hsa_kernel_class_time(ctypes.Structure):
    _fields_ = [("calls", ctypes.c_uint64), ("ms", ctypes.c_double), ("work", ctypes.c_double)]


KERNEL_CLASSES = ("attention", "gemm", "rows", "tokens")


class hsa_state(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("v_hat", ctypes.c_void_p),
                ("v_hat_prev", ctypes.c_void_p), ("v_fresh", ctypes.c_void_p),
                ("score", ctypes.c_void_p), ("g", ctypes.c_void_p), ("mask", ctypes.c_void_p),
                ("active_idx", ctypes.c_void_p), ("h", ctypes.c_void_p),
                ("k_cache", ctypes.POINTER(ctypes.c_void_p)),
                ("v_cache", ctypes.POINTER(ctypes.c_void_p))]


_lib = None


def load() -> ctypes.CDLL:
    """Load libhsa.so (built in-tree by ``token_sparse_denoising_layer_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m token_sparse_denoising_layer_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sig = {
        "hsa_create": (I, [ctypes.POINTER(hsa_model_cfg), I, ctypes.POINTER(I), ctypes.POINTER(I),
                           I, I, P, ctypes.POINTER(P)]),
        "hsa_destroy": (None, [P]),
        "hsa_last_error": (ctypes.c_char_p, [P]),
        "hsa_set_stream": (I, [P, P]),
        "hsa_sync_check": (I, [P]),
        "hsa_selftest_timeout": (I, [P, I]),
        "hsa_kernel_launches": (ctypes.c_uint64, [P]),
        "hsa_time_kernels": (I, [P, I]),
        "hsa_kernel_times": (I, [P, ctypes.POINTER(hsa_kernel_class_time), I]),
        "hsa_n_active": (I, [P, I]),
        "hsa_schedule": (I, [P, I, P, P, P, P, ctypes.POINTER(I)]),
        "hsa_score": (I, [P, P, P, P]),
        "hsa_select_from_score": (I, [P, P, P]),
        "hsa_select_groups": (I, [P, P, P, P, P]),
        "hsa_ln_gather": (I, [P, P, P, I, P]),
        "hsa_qkv_project": (I, [P, P, P, P, I, P, P, P]),
        "hsa_qkv_project_peers": (I, [P, P, P, P, I, P, ctypes.POINTER(P), ctypes.POINTER(P), I]),
        "hsa_linear": (I, [P, P, I, I, P, I, P]),
        "hsa_kv_scatter": (I, [P, P, P, P, I, P, P]),
        "hsa_kv_scatter_packed": (I, [P, P, P, I, P, P]),
        "hsa_attention": (I, [P, P, I, P, P, P]),
        "hsa_attention_kv": (I, [P, P, I, P, P, I, P]),
        "hsa_out_proj_residual": (I, [P, P, P, P, I, P]),
        "hsa_mlp_residual": (I, [P, P, P, P, P, I]),
        "hsa_ln_gather_mod": (I, [P, P, P, I, P, P, P]),
        "hsa_out_proj_residual_gated": (I, [P, P, P, P, I, P, P]),
        "hsa_mlp_residual_mod": (I, [P, P, P, P, P, I, P, P, P]),
        "hsa_layer_forward": (I, [P, ctypes.POINTER(hsa_layer_weights), P, P, I, P, P]),
        "hsa_layer_forward_cond": (I, [P, ctypes.POINTER(hsa_layer_weights), P,
                                       ctypes.POINTER(hsa_cross_attn), P, P, I, P, P]),
        "hsa_embed": (I, [P, P, P, P, I, P]),
        "hsa_head": (I, [P, P, P, P, I, P]),
        "hsa_euler_step": (I, [P, P, P, P, P, P, F, F]),
        "hsa_euler_step_score": (I, [P, P, P, P, P, P, F, F, P]),
        "hsa_step": (I, [P, ctypes.POINTER(hsa_model_weights), ctypes.POINTER(hsa_state), I, F, F, I]),
        "hsa_step_cond": (I, [P, ctypes.POINTER(hsa_model_weights), ctypes.POINTER(hsa_state),
                              ctypes.POINTER(hsa_cond), I, F, F, I]),
        "hsa_select_groups_static": (I, [P, P, I, ctypes.POINTER(I), I, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(t) -> Optional[int]:
    """Device address of a tensor (None passes NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libhsa takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libhsa takes contiguous tensors")
    return t.data_ptr()


def _addr(t) -> Optional[int]:
    """Device address of a tensor, or an int taken as a device address as is."""
    if isinstance(t, int):
        return t
    return _p(t)


def _check(ctx, status: int) -> None:
    if status != 0:
        msg = load().hsa_last_error(ctx)
        raise HsaError(status, msg.decode() if msg else "")


class Context:
    """Owns an ``hsa_ctx*``; the handle is ``.ptr``.  Destroyed with ``close()`` or on GC."""

    def __init__(self, ptr: int, cfg: hsa_model_cfg):
        self.ptr = ptr
        self.cfg = cfg

    def close(self) -> None:
        if self.ptr:
            load().hsa_destroy(self.ptr)
            self.ptr = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return getattr(stream, "cuda_stream", stream) or None


def hsa_create(N: int, D: int, H: int, F: int, L: int, T: int, budgets: Sequence[int],
               counts: Sequence[int], m: int = 0, C: int = 16, stream=None) -> Context:
    lib = load()
    K = len(budgets)
    cfg = hsa_model_cfg(N, C, D, H, F, L)
    b = (ctypes.c_int * K)(*budgets)
    c = (ctypes.c_int * K)(*counts)
    out = ctypes.c_void_p()
    st = lib.hsa_create(ctypes.byref(cfg), T, b, c, K, m, _stream_ptr(stream), ctypes.byref(out))
    _check(None, st)
    return Context(out.value, cfg)


def hsa_destroy(ctx: Context) -> None:
    ctx.close()


def hsa_set_stream(ctx: Context, stream) -> None:
    _check(ctx.ptr, load().hsa_set_stream(ctx.ptr, _stream_ptr(stream)))


def hsa_sync_check(ctx: Context) -> None:
    _check(ctx.ptr, load().hsa_sync_check(ctx.ptr))


def hsa_selftest_timeout(ctx: Context, timeout_us: int) -> None:
    _check(ctx.ptr, load().hsa_selftest_timeout(ctx.ptr, timeout_us))


def hsa_kernel_launches(ctx: Context) -> int:
    return int(load().hsa_kernel_launches(ctx.ptr))


def hsa_time_kernels(ctx: Context, on: bool) -> None:
    _check(ctx.ptr, load().hsa_time_kernels(ctx.ptr, 1 if on else 0))


def hsa_kernel_times(ctx: Context) -> dict:
    """Per-class totals since timing was turned on or last read: {class:
    {"calls", "ms", "work"}} (work: FLOP for attention and GEMM, bytes for row
    kernels); reading clears them."""
    out = (hsa_kernel_class_time * len(KERNEL_CLASSES))()
    _check(ctx.ptr, load().hsa_kernel_times(ctx.ptr, out, len(KERNEL_CLASSES)))
    return {name: {"calls": int(out[k].calls), "ms": float(out[k].ms), "work": float(out[k].work)}
            for k, name in enumerate(KERNEL_CLASSES)}


def hsa_n_active(ctx: Context, i: int) -> int:
    return load().hsa_n_active(ctx.ptr, i)


def hsa_schedule(ctx: Context, i: int, g, mask, active_idx, n_active_dev=None) -> int:
    n = ctypes.c_int(0)
    _check(ctx.ptr, load().hsa_schedule(ctx.ptr, i, _p(g), _p(mask), _p(active_idx),
                                        _p(n_active_dev), ctypes.byref(n)))
    return n.value


def hsa_score(ctx: Context, v_prev, v_cur, score) -> None:
    _check(ctx.ptr, load().hsa_score(ctx.ptr, _p(v_prev), _p(v_cur), _p(score)))


def hsa_select_from_score(ctx: Context, score, g) -> None:
    _check(ctx.ptr, load().hsa_select_from_score(ctx.ptr, _p(score), _p(g)))


def hsa_select_groups(ctx: Context, v_prev, v_cur, score, g) -> None:
    _check(ctx.ptr, load().hsa_select_groups(ctx.ptr, _p(v_prev), _p(v_cur), _p(score), _p(g)))


def hsa_ln_gather(ctx: Context, x, idx, n: int, u) -> None:
    _check(ctx.ptr, load().hsa_ln_gather(ctx.ptr, _p(x), _p(idx), n, _p(u)))


def hsa_qkv_project(ctx: Context, w_qkv, u, idx, n: int, q, k_cache, v_cache) -> None:
    _check(ctx.ptr, load().hsa_qkv_project(ctx.ptr, _p(w_qkv), _p(u), _p(idx), n, _p(q),
                                           _p(k_cache), _p(v_cache)))


def hsa_qkv_project_peers(ctx: Context, w_qkv, u, idx, n: int, q, k_caches, v_caches) -> None:
    """hsa_qkv_project writing the fresh K/V rows into every cache of the lists.

    ``k_caches`` / ``v_caches`` are equal-length sequences of device buffers
    (tensors) or raw device addresses (ints, e.g. peers' caches mapped into this
    process by CUDA IPC)."""
    if len(k_caches) != len(v_caches):
        raise ValueError("k_caches and v_caches differ in length")
    G = len(k_caches)
    ks = (ctypes.c_void_p * max(G, 1))(*[_addr(t) for t in k_caches])
    vs = (ctypes.c_void_p * max(G, 1))(*[_addr(t) for t in v_caches])
    _check(ctx.ptr, load().hsa_qkv_project_peers(ctx.ptr, _p(w_qkv), _p(u), _p(idx), n, _p(q),
                                                 ks, vs, G))


def hsa_linear(ctx: Context, a, M: int, Kd: int, w, Ncols: int, out) -> None:
    _check(ctx.ptr, load().hsa_linear(ctx.ptr, _p(a), M, Kd, _p(w), Ncols, _p(out)))


def hsa_kv_scatter(ctx: Context, k_rows, v_rows, idx, n: int, k_cache, v_cache) -> None:
    _check(ctx.ptr, load().hsa_kv_scatter(ctx.ptr, _p(k_rows), _p(v_rows), _p(idx), n,
                                          _p(k_cache), _p(v_cache)))


def hsa_kv_scatter_packed(ctx: Context, kv_rows, idx, n: int, k_cache, v_cache) -> None:
    _check(ctx.ptr, load().hsa_kv_scatter_packed(ctx.ptr, _p(kv_rows), _p(idx), n, _p(k_cache),
                                                 _p(v_cache)))


def hsa_attention(ctx: Context, q, n: int, k_cache, v_cache, o) -> None:
    _check(ctx.ptr, load().hsa_attention(ctx.ptr, _p(q), n, _p(k_cache), _p(v_cache), _p(o)))


def hsa_attention_kv(ctx: Context, q, n: int, k, v, n_kv: int, o) -> None:
    _check(ctx.ptr, load().hsa_attention_kv(ctx.ptr, _p(q), n, _p(k), _p(v), n_kv, _p(o)))


def hsa_out_proj_residual(ctx: Context, w_o, o, idx, n: int, x) -> None:
    _check(ctx.ptr, load().hsa_out_proj_residual(ctx.ptr, _p(w_o), _p(o), _p(idx), n, _p(x)))


def hsa_mlp_residual(ctx: Context, w_1, w_2, x, idx, n: int) -> None:
    _check(ctx.ptr, load().hsa_mlp_residual(ctx.ptr, _p(w_1), _p(w_2), _p(x), _p(idx), n))


def _opt(t):
    return _p(t) if t is not None else None


def hsa_ln_gather_mod(ctx: Context, x, idx, n: int, u, shift=None, scale=None) -> None:
    _check(ctx.ptr, load().hsa_ln_gather_mod(ctx.ptr, _p(x), _p(idx), n, _p(u), _opt(shift),
                                             _opt(scale)))


def hsa_out_proj_residual_gated(ctx: Context, w_o, o, idx, n: int, x, gate=None) -> None:
    _check(ctx.ptr, load().hsa_out_proj_residual_gated(ctx.ptr, _p(w_o), _p(o), _p(idx), n,
                                                       _p(x), _opt(gate)))


def hsa_mlp_residual_mod(ctx: Context, w_1, w_2, x, idx, n: int, shift=None, scale=None,
                         gate=None) -> None:
    _check(ctx.ptr, load().hsa_mlp_residual_mod(ctx.ptr, _p(w_1), _p(w_2), _p(x), _p(idx), n,
                                                _opt(shift), _opt(scale), _opt(gate)))


def layer_weights(w_qkv, w_o, w_1, w_2) -> hsa_layer_weights:
    """The struct holds raw device addresses, so it also keeps the tensors alive."""
    s = hsa_layer_weights(_p(w_qkv), _p(w_o), _p(w_1), _p(w_2))
    s._keep = (w_qkv, w_o, w_1, w_2)
    return s


def hsa_layer_forward(ctx: Context, w: hsa_layer_weights, x, idx, n: int, k_cache, v_cache) -> None:
    _check(ctx.ptr, load().hsa_layer_forward(ctx.ptr, ctypes.byref(w), _p(x), _p(idx), n,
                                             _p(k_cache), _p(v_cache)))


def cross_attn(w_q, w_o, k_txt, v_txt, n_txt: int) -> hsa_cross_attn:
    """The struct holds raw device addresses, so it also keeps the tensors alive."""
    s = hsa_cross_attn(_p(w_q), _p(w_o), _p(k_txt), _p(v_txt), n_txt)
    s._keep = (w_q, w_o, k_txt, v_txt)
    return s


def hsa_layer_forward_cond(ctx: Context, w: hsa_layer_weights, mod, xa, x, idx, n: int, k_cache,
                           v_cache) -> None:
    """mod: device fp32 [6, D] or None;  xa: hsa_cross_attn or None."""
    _check(ctx.ptr, load().hsa_layer_forward_cond(
        ctx.ptr, ctypes.byref(w), _p(mod) if mod is not None else None,
        ctypes.byref(xa) if xa is not None else None, _p(x), _p(idx), n, _p(k_cache),
        _p(v_cache)))


def hsa_embed(ctx: Context, w_in, x_lat, idx, n: int, h) -> None:
    _check(ctx.ptr, load().hsa_embed(ctx.ptr, _p(w_in), _p(x_lat), _p(idx), n, _p(h)))


def hsa_head(ctx: Context, w_head, h, idx, n: int, v_fresh) -> None:
    _check(ctx.ptr, load().hsa_head(ctx.ptr, _p(w_head), _p(h), _p(idx), n, _p(v_fresh)))


def hsa_euler_step(ctx: Context, x, v_hat, v_hat_prev, v_fresh, mask, sigma_i: float,
                   sigma_next: float) -> None:
    _check(ctx.ptr, load().hsa_euler_step(ctx.ptr, _p(x), _p(v_hat), _p(v_hat_prev), _p(v_fresh),
                                          _p(mask), float(sigma_i), float(sigma_next)))


def hsa_euler_step_score(ctx: Context, x, v_hat, v_hat_prev, v_fresh, mask, sigma_i: float,
                         sigma_next: float, score) -> None:
    _check(ctx.ptr, load().hsa_euler_step_score(ctx.ptr, _p(x), _p(v_hat), _p(v_hat_prev),
                                                _p(v_fresh), _p(mask), float(sigma_i),
                                                float(sigma_next), _p(score)))


class ModelBinding:
    """Keeps the ctypes structs of hsa_step (weights and state) alive."""

    def __init__(self, w_in, w_head, layers, x, v_hat, v_hat_prev, v_fresh, score, g, mask,
                 active_idx, h, k_caches, v_caches):
        L = len(layers)
        self._layers = (hsa_layer_weights * max(L, 1))(*[layer_weights(*lw) for lw in layers])
        self.weights = hsa_model_weights(_p(w_in), _p(w_head), self._layers)
        self._kc = (ctypes.c_void_p * max(L, 1))(*[_p(t) for t in k_caches])
        self._vc = (ctypes.c_void_p * max(L, 1))(*[_p(t) for t in v_caches])
        self.state = hsa_state(_p(x), _p(v_hat), _p(v_hat_prev), _p(v_fresh), _p(score), _p(g),
                               _p(mask), _p(active_idx), _p(h), self._kc, self._vc)
        self._keep = (w_in, w_head, layers, x, v_hat, v_hat_prev, v_fresh, score, g, mask,
                      active_idx, h, k_caches, v_caches)


def hsa_step(ctx: Context, model: ModelBinding, i: int, sigma_i: float, sigma_next: float,
             regroup: bool = True) -> None:
    _check(ctx.ptr, load().hsa_step(ctx.ptr, ctypes.byref(model.weights), ctypes.byref(model.state),
                                    i, float(sigma_i), float(sigma_next), 1 if regroup else 0))


class StepCond:
    """The ctypes arrays of one iteration's conditioning (keeps them alive).

    mods: a list of L device fp32 [6, D] tensors (None entries allowed) or
    None; cross: a list of L hsa_cross_attn structs (see cross_attn) or None."""

    def __init__(self, mods=None, cross=None):
        self._mods = None if mods is None else (ctypes.c_void_p * max(len(mods), 1))(
            *[None if m is None else _p(m) for m in mods])
        self._cross = None if cross is None else (hsa_cross_attn * max(len(cross), 1))(*cross)
        self.struct = hsa_cond(
            ctypes.cast(self._mods, ctypes.POINTER(ctypes.c_void_p)) if mods is not None else None,
            ctypes.cast(self._cross, ctypes.POINTER(hsa_cross_attn)) if cross is not None else None)
        self._keep = (mods, cross)


def hsa_step_cond(ctx: Context, model: ModelBinding, cond: Optional[StepCond], i: int,
                  sigma_i: float, sigma_next: float, regroup: bool = True) -> None:
    _check(ctx.ptr, load().hsa_step_cond(
        ctx.ptr, ctypes.byref(model.weights), ctypes.byref(model.state),
        ctypes.byref(cond.struct) if cond is not None else None, i, float(sigma_i),
        float(sigma_next), 1 if regroup else 0))


def hsa_select_groups_static(v_prev, v_cur, N: int, counts: Sequence[int], g, stream=None) -> None:
    """Group selection without a context or any device allocation (see include/hsa.h).

    Its scratch is one static device array of the library, sized for at most
    SELECT_STATIC_MAX_N tokens; concurrent calls on the GPU race on it.
    """
    K = len(counts)
    c = (ctypes.c_int * K)(*counts)
    st = load().hsa_select_groups_static(_p(v_prev), _p(v_cur), N, c, K, _p(g), _stream_ptr(stream))
    if st != 0:
        why = {8: f"N = {N} exceeds the static scratch limit of {SELECT_STATIC_MAX_N} tokens"}
        raise HsaError(st, why.get(st, "hsa_select_groups_static rejected its arguments"))
