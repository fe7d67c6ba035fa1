"""bit_kv_cache_22_b200 -- decode attention over a KIVI-style low-bit KV cache on B200.

The compute path is the CUDA library ``libkvq.so`` (sm_100a kernels behind a
C ABI declared in ``include/kvq.h``); the Python side only marshals tensors.
"""
from . import workloads  # noqa: F401  (seeded synthetic inputs, no method arithmetic)

__all__ = ["workloads"]
