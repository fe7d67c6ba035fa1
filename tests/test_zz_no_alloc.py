"""The allocation-free decode entry point (kvq_decode_attention_noalloc).

Some callers cannot allocate device memory at decode time -- code that runs
while another framework owns every allocation on the device, plugin hosts
that forbid cudaMalloc, latency-bound loops that must stay off the allocator.
For them the library keeps the per-split partials in a fixed 4 MiB static
device array instead of a caller-provided workspace.  These tests call it
through the C ABI and check that it returns what kvq_decode_attention returns
and what the CPU oracle returns, within the tolerance of the other parity
tests, on two calls in a row -- also when a call with many splits on one cache
is followed on the same stream by a call with few splits on a cache of another
shape, which reads less of the shared array than the first one wrote.  The
file is collected last so that a run stopping at its first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

import kvq_testlib as tl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _noalloc(cache: kvq.KVQCache, q: torch.Tensor, out: torch.Tensor) -> int:
    lib = kvq.load()
    return lib.kvq_decode_attention_noalloc(cache._h, q.data_ptr(), out.data_ptr(),
                                            torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name", ["gqa8b", "llama7b", "tiny"])
def test_noalloc_matches_workspace_decode_twice(name):
    base = wl.WORKLOADS[name]
    w = base if name == "tiny" else base.replace(B=2, Hkv=min(base.Hkv, 4),
                                                 Hq=base.g * min(base.Hkv, 4),
                                                 T=3 * base.R + 17, steps=3)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    cache = tl.new_cache(w)
    ref = tl.new_oracle(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)
    for s in range(2):                       # two calls in a row, different queries and lengths
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        ref.append(tK[s], tV[s])
        q = tl.to_dev(tQ[s], w)
        want = cache.decode_attention(q).cpu().numpy().astype(np.float64)
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(cache, q, out) == kvq.KVQ_OK, kvq.load().kvq_last_error()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        tl.assert_close(got, want, f"{name} call {s}")
        tl.assert_close(got, ref.decode(tQ[s]), f"{name} call {s} against the oracle")


def test_noalloc_two_caches_of_different_shape_back_to_back():
    """A decode with many splits on one cache, then on the same stream a decode with
    fewer splits on a cache of another shape: the second reads only partials it wrote."""
    big = wl.WORKLOADS["gqa8b"].replace(B=2, Hkv=2, Hq=8, T=40 * 128 + 9, steps=1)
    small = wl.WORKLOADS["llama7b"].replace(B=1, Hkv=3, Hq=3, T=128 + 5, steps=1)
    caches, refs, qs = [], [], []
    for w in (big, small):
        XK, XV = wl.prefill_bits(w)
        _, _, tQ = wl.decode_bits(w)
        c, r = tl.new_cache(w), tl.new_oracle(w)
        c.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
        r.prefill(XK, XV)
        caches.append(c)
        refs.append(r)
        qs.append(tQ[0])
    assert caches[0].splits() > caches[1].splits()
    for rep in range(2):
        outs = []
        for w, c, q in zip((big, small), caches, qs):
            out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
            assert _noalloc(c, tl.to_dev(q, w), out) == kvq.KVQ_OK, kvq.load().kvq_last_error()
            outs.append(out)
        for w, r, q, out in zip((big, small), refs, qs, outs):
            tl.assert_close(out.cpu().numpy(), r.decode(q), f"{w.name} round {rep}")


def test_noalloc_rejects_a_decode_beyond_its_scratch():
    # 256 x 32 query heads of d=128 need > 4 MiB of partials even with one split
    w = wl.WORKLOADS["gqa8b"].replace(B=256, T=64, steps=1, R=32)
    XK, XV = wl.prefill_bits(w)
    _, _, tQ = wl.decode_bits(w)
    cache = tl.new_cache(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    q = tl.to_dev(tQ[0], w)
    out = torch.zeros((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    launches = kvq.kernel_launches()
    assert _noalloc(cache, q, out) == kvq.KVQ_ERR_CAPACITY
    assert b"static scratch" in kvq.load().kvq_last_error()
    assert kvq.kernel_launches() == launches
    assert torch.count_nonzero(out) == 0
