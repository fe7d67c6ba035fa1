"""GPU parity of LogQuant retention ("Resumo Técnico: LogQuant", sections 2 and 4):
the library's LogQuant cache against the oracle's on the same seeded inputs.  The
retained positions must be the oracle's, the quantized blocks bit-exact, outputs
|gpu - ref| <= 2e-3 + 1e-2 |ref|."""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

import kvq_testlib as tl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def new_lq(w: wl.Workload, W: int, capacity: int) -> kvq.KVQCache:
    return kvq.KVQCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, tl.torch_dtype(w),
                        capacity, "cuda", window=W)


def new_lq_oracle(w: wl.Workload, W: int):
    return oracle.LogQuantCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, W, w.bits, w.symmetric, w.dtype)


def check_state(cache, ref, w):
    assert cache.state() == (ref.Tq, len(ref.F))
    assert cache.retained() == ref.F
    tl.assert_codes_equal(tl.gpu_packed(cache, ref.Tq), ref.packed(), w.symmetric)


# (workload, changes, W): the tensor-core kernel with 1, 2 and 4 query heads per kv head,
# 4-bit groups of 128, the CUDA-core kernel (16-token key groups), the symmetric variant, fp16
CASES = [
    ("tiny", dict(), 32),
    ("llama7b", dict(B=2, Hq=2, Hkv=2, T=900), 128),
    ("gqa8b", dict(B=2, Hq=8, Hkv=2, T=700), 64),
    ("gqa8b", dict(B=2, Hq=4, Hkv=2, T=500, Gv=64), 32),
    ("stream2", dict(B=2, Hq=4, Hkv=2, G=16, Gv=16, T=333), 48),
    ("stream4sym", dict(B=2, Hq=8, Hkv=2, T=420), 64),
]


@pytest.mark.parametrize("name,changes,W", CASES)
def test_logquant_episode_matches_oracle(name, changes, W):
    w = wl.WORKLOADS[name].replace(**changes)
    steps = 2 * W + 7                          # at least two retention events during decode
    w = w.replace(steps=steps)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    cap = -(-(w.T + steps) // W) * W
    cache = new_lq(w, W, cap)
    ref = new_lq_oracle(w, W)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)
    check_state(cache, ref, w)
    for s in range(steps):
        blocks = len(ref.blocks)
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        ref.append(tK[s], tV[s])
        if len(ref.blocks) != blocks:
            check_state(cache, ref, w)
        if s % 6 == 0 or s == steps - 1:
            out = cache.decode_attention(tl.to_dev(tQ[s], w)).cpu().numpy()
            tl.assert_close(out, ref.decode(tQ[s]), f"{name} W={W} step {s}")
    check_state(cache, ref, w)
    cache.check_device()


def test_logquant_fused_append_decode_equals_separate_calls():
    w = wl.WORKLOADS["gqa8b"].replace(B=2, Hq=8, Hkv=2, T=300, steps=80)
    W = 32
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    a, b = new_lq(w, W, 512), new_lq(w, W, 512)
    for c in (a, b):
        c.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    for s in range(w.steps):
        oa = a.append_decode(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w), tl.to_dev(tQ[s], w))
        b.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        ob = b.decode_attention(tl.to_dev(tQ[s], w))
        assert a.state() == b.state() and a.retained() == b.retained()
        assert torch.equal(oa, ob), f"step {s}"


def test_logquant_prefill_then_appends_equals_longer_prefill_on_gpu():
    w = wl.WORKLOADS["stream2"].replace(B=2, Hq=8, Hkv=2, T=400)
    W = 32
    XK, XV = wl.prefill_bits(w, T=w.T + 50)
    a, b = new_lq(w, W, 512), new_lq(w, W, 512)
    a.prefill_quantize(tl.to_dev(XK[:, :, :w.T], w), tl.to_dev(XV[:, :, :w.T], w))
    for t in range(w.T, w.T + 50):
        a.append(tl.to_dev(np.ascontiguousarray(XK[:, :, t]), w), tl.to_dev(np.ascontiguousarray(XV[:, :, t]), w))
    b.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    assert a.state() == b.state() and a.retained() == b.retained()
    Tq = a.state()[0]
    tl.assert_codes_equal(tl.gpu_packed(a, Tq), tl.gpu_packed(b, Tq), w.symmetric)
    _, _, tQ = wl.decode_bits(w)
    oa = a.decode_attention(tl.to_dev(tQ[0], w))
    ob = b.decode_attention(tl.to_dev(tQ[0], w))
    assert torch.equal(oa, ob)


def test_logquant_capacity_and_state_errors():
    w = wl.WORKLOADS["tiny"]
    W = 32
    cache = new_lq(w, W, 96)                  # rounds up to 96 = 3W: three blocks
    X = torch.zeros(w.B, w.Hkv, 3 * W + 3 * W - 1, w.d, dtype=torch.float16, device="cuda")
    cache.prefill_quantize(X, X)             # 191 tokens: 3 blocks leave, 95 stay
    assert cache.state() == (96, 95)
    t = torch.zeros(w.B, w.Hkv, w.d, dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KVQError):
        cache.append(t, t)                   # a fourth block would pass the capacity
    assert cache.state() == (96, 95)
    plain = tl.new_cache(w)
    with pytest.raises(kvq.KVQError):
        plain.retained()
