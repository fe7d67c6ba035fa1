"""bit_kv_cache_22_b200 -- decode attention over a KIVI-style low-bit KV cache on B200.

The compute path is the CUDA library ``libkvq.so`` (sm_100a kernels behind the
C ABI declared in ``include/kvq.h``); :mod:`.kvq` only marshals tensors into it.
"""
from . import workloads  # noqa: F401  (seeded synthetic inputs, no method arithmetic)
from .kvq import (KVQCache, KVQError, append, decode_attention, load,  # noqa: F401
                  prefill_quantize)

__all__ = ["KVQCache", "KVQError", "prefill_quantize", "append", "decode_attention", "load",
           "workloads"]
