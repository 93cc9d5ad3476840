"""Helpers for the GPU parity tests: device copies and the error metrics."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from token_sparse_denoising_layer_b200 import abi  # noqa: E402


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    abi.load()   # fails loudly if libhsa.so is missing


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bf(a):
    """float32 numpy (bf16-representable) -> CUDA bf16 tensor."""
    return dev(np.asarray(a, dtype=np.float32), torch.bfloat16)


def host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def normwise(gpu, ref):
    """max|gpu - ref| / max|ref| (the bf16 tolerance metric)."""
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(np.asarray(gpu, dtype=np.float64) - ref).max() / max(np.abs(ref).max(), 1e-30))


BF16_TOL = 1e-2     # layer and attention outputs, fp32 accumulation
EULER_TOL = 1e-5    # fp32 cached Euler vs float64
