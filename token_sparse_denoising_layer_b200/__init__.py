"""HSA (Heterogeneous Step Allocation) denoising step for NVIDIA B200 (sm_100a).

The compute path is libhsa.so (hand-written CUDA kernels behind the C ABI in
include/hsa.h); ``abi`` is its thin ctypes binding and ``synth`` makes seeded
synthetic workloads.  Build the library with
``python -m token_sparse_denoising_layer_b200.build``.
"""

from . import abi  # noqa: F401

__all__ = ["abi", "synth", "build"]
