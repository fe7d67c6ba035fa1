"""Magnitude range of the decode path, through the C ABI against the oracle.

The decode kernels carry q s and p s on the tensor cores in bf16 times fixed powers of two
(section 核心公式 / 量化基础 of "Atom: Low-bit Quantization for Efficient and Accurate LLM
Serving" gives the scales; the powers of two are this library's).  They serve scales up to
2^31; a larger scale is still quantized exactly but raises a status bit that
kvq_check_device reports.  Both ends of the served range are compared with the oracle
after dividing out the common power of two, so the usual tolerance keeps its meaning.
"""
import numpy as np
import pytest
import torch

from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

import kvq_testlib as tl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _episode(w, k_mult, v_mult, steps=3):
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    scale = lambda bits, m: wl.to_bits(wl.from_bits(bits, w.dtype) * np.float32(m), w.dtype)
    XK, XV, tK, tV = scale(XK, k_mult), scale(XV, v_mult), scale(tK, k_mult), scale(tV, v_mult)
    cache, ref = tl.new_cache(w), tl.new_oracle(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)
    outs = []
    for s in range(steps):
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        ref.append(tK[s], tV[s])
        got = cache.decode_attention(tl.to_dev(tQ[s], w)).cpu().numpy().astype(np.float64)
        outs.append((got, ref.decode(tQ[s])))
    return cache, ref, outs


# the contiguous kernels (g = 4 and g = 1), 2- and 4-bit, symmetric
GEOMS = [("gqa8b", {}), ("llama7b", {}), ("stream4sym", {})]


@pytest.mark.parametrize("name,extra", GEOMS)
@pytest.mark.parametrize("k_mult,v_mult", [(2.0 ** 20, 2.0 ** 29), (2.0 ** -30, 2.0 ** -30), (1.0, 2.0 ** -33)])
def test_both_ends_of_the_served_range(name, extra, k_mult, v_mult):
    base = wl.WORKLOADS[name]
    w = base.replace(B=2, Hkv=2, Hq=2 * base.g, T=2 * base.R + 19, steps=3, **extra)
    cache, _, outs = _episode(w, k_mult, v_mult)
    for s, (got, want) in enumerate(outs):
        tl.assert_close(got / v_mult, want / v_mult, f"{name} k x{k_mult:g} v x{v_mult:g} step {s}")
    cache.check_device()                                # nothing outside the served range


@pytest.mark.parametrize("name", ["gqa8b", "llama7b"])
@pytest.mark.parametrize("which", ["keys", "values"])
def test_scales_beyond_the_range_are_reported(name, which):
    base = wl.WORKLOADS[name]
    w = base.replace(B=1, Hkv=2, Hq=2 * base.g, T=base.R + 7, steps=1)
    k_mult, v_mult = (2.0 ** 36, 1.0) if which == "keys" else (1.0, 2.0 ** 36)
    cache, ref, _ = _episode(w, k_mult, v_mult, steps=1)
    # the codes, scales and zeros are still exact
    tl.assert_codes_equal(tl.gpu_packed(cache, ref.Tq), ref.packed(), w.symmetric)
    with pytest.raises(kvq.KVQError) as ei:
        cache.check_device()
    assert ei.value.status == kvq.KVQ_ERR_DEVICE_CHECK
    assert b"scale" in kvq.load().kvq_last_error()
    cache.check_device()                                # the word was cleared
