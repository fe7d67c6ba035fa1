"""Every decode kernel a cache can be switched to (kvq_set_decode_kernel) against the oracle.

The three kernels read the same packed layout: decode_split_kernel on CUDA cores,
decode_tc_kernel with integer mma.sync for keys, decode_mma_kernel with bf16 mma.sync for
keys and values.  Each is compared with the oracle on the same cache, step by step, for
the grouped-query and the MHA geometry, 2- and 4-bit, with key groups of one item (2
tiles) and of several.
"""
import numpy as np
import pytest
import torch

from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

import kvq_testlib as tl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

KERNELS = [kvq.KVQ_DECODE_CUDA_CORES, kvq.KVQ_DECODE_INT8_MMA, kvq.KVQ_DECODE_BF16_MMA, kvq.KVQ_DECODE_AUTO]
GEOMS = [
    ("gqa8b", dict(B=2, Hkv=2, Hq=8, T=9 * 128 + 40)),                    # G = 32: one item per group
    ("gqa8b", dict(B=2, Hkv=2, Hq=8, T=9 * 128 + 40, G=64, Gv=64)),       # G = 64
    ("llama7b", dict(B=2, Hkv=3, Hq=3, T=7 * 128 + 77)),                  # 4-bit, G = 128
    ("stream4sym", dict(B=1, Hkv=2, Hq=4, T=5 * 128 + 3)),                # symmetric, HG = 2
]


@pytest.mark.parametrize("name,extra", GEOMS)
def test_every_kernel_matches_the_oracle(name, extra):
    w = wl.WORKLOADS[name].replace(steps=3, **extra)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    cache, ref = tl.new_cache(w), tl.new_oracle(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)
    for s in range(w.steps):
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        ref.append(tK[s], tV[s])
        want = ref.decode(tQ[s])
        q = tl.to_dev(tQ[s], w)
        for k in KERNELS:
            cache.set_decode_kernel(k)
            got = cache.decode_attention(q).cpu().numpy().astype(np.float64)
            tl.assert_close(got, want, f"{name} {extra} kernel {k} step {s}")
    cache.check_device()


def test_unsupported_choices_are_refused():
    w = wl.WORKLOADS["gqa8b"].replace(B=1, Hkv=1, Hq=8, T=256, steps=1)   # 8 query heads per kv head
    cache = tl.new_cache(w)
    for k in (kvq.KVQ_DECODE_INT8_MMA, kvq.KVQ_DECODE_BF16_MMA):
        with pytest.raises(kvq.KVQError) as ei:
            cache.set_decode_kernel(k)
        assert ei.value.status == kvq.KVQ_ERR_UNSUPPORTED
    with pytest.raises(kvq.KVQError) as ei:
        cache.set_decode_kernel(7)
    assert ei.value.status == kvq.KVQ_ERR_INVALID_ARG
    cache.set_decode_kernel(kvq.KVQ_DECODE_CUDA_CORES)
    cache.set_decode_kernel(kvq.KVQ_DECODE_AUTO)
