"""The C-ABI library on the host (no GPU): it loads, exports every symbol the
header declares, and rejects bad arguments on the host before any CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest

from token_sparse_denoising_layer_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "hsa.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hsa_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(abi.LIB_PATH):
        from token_sparse_denoising_layer_b200 import build
        build.build()
    return abi.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert len(declared) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    assert sorted(abi.SYMBOLS) == declared
    for s in declared:
        assert getattr(lib, s) is not None


def _create(lib, N=256, C=16, D=128, H=2, F=512, L=1, T=8, budgets=(8, 4), counts=(128, 128), m=0):
    cfg = abi.hsa_model_cfg(N, C, D, H, F, L)
    K = len(budgets)
    out = ctypes.c_void_p(123)
    st = lib.hsa_create(ctypes.byref(cfg), T, (ctypes.c_int * K)(*budgets),
                        (ctypes.c_int * K)(*counts), K, m, None, ctypes.byref(out))
    return st, out.value, lib.hsa_last_error(None).decode()


@pytest.mark.parametrize("kw,status,word", [
    (dict(budgets=(8, 3), counts=(128, 128)), 2, "divide"),
    (dict(budgets=(4, 2), counts=(128, 128)), 2, "s_1"),
    (dict(budgets=(8, 8), counts=(128, 128)), 2, "decreasing"),
    (dict(counts=(100, 100)), 2, "sum to N"),
    (dict(C=8), 3, "C == 16"),
    (dict(D=96, H=1), 3, "D % 128"),
    (dict(D=384, H=2), 3, "head_dim"),
    (dict(F=100), 3, "F % 64"),
    (dict(m=5), 1, "phase window"),
    (dict(budgets=tuple(range(9, 0, -1)), T=9, counts=(256,) + (0,) * 8), 1, "K must"),
])
def test_create_rejects_on_host(lib, kw, status, word):
    st, ptr, msg = _create(lib, **kw)
    assert st == status
    assert ptr is None
    assert word in msg


def test_null_context_is_rejected(lib):
    assert lib.hsa_euler_step(None, None, None, None, None, None, 0.0, 1.0) == 1
    assert lib.hsa_n_active(None, 0) == -1
    lib.hsa_destroy(None)


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(abi, "_lib", None)
    monkeypatch.setattr(abi, "LIB_PATH", "/nonexistent/libhsa.so")
    with pytest.raises(RuntimeError, match="missing"):
        abi.load()

