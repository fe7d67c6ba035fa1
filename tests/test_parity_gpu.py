"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same
seeded inputs.  Codes, scales and zeros must match bit for bit; attention
outputs must satisfy |gpu - ref| <= 2e-3 + 1e-2 |ref| elementwise."""
import numpy as np
import pytest
import torch

from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

import kvq_testlib as tl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ALL = list(wl.WORKLOADS)


def reduced(w: wl.Workload) -> wl.Workload:
    """Same quantiser, head size and distributions; a batch of 2, at most 2 kv
    heads, a ragged prompt (2R + 40 tokens) and enough steps to cross a flush."""
    if w.name == "tiny":
        return w.replace(steps=w.R + 12)
    Hkv = min(w.Hkv, 2)
    return w.replace(B=2, Hkv=Hkv, Hq=w.g * Hkv, T=2 * w.R + 40, steps=w.R + 20)


def run_episode(w: wl.Workload, check_every=1, split_limit=None):
    """Prefill + all decode steps on GPU and oracle; compare along the way."""
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    cache = tl.new_cache(w)
    if split_limit:
        cache.set_split_limit(split_limit)
    ref = tl.new_oracle(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)
    assert cache.state() == (ref.Tq, ref.r)
    tl.assert_codes_equal(tl.gpu_packed(cache, ref.Tq), ref.packed(), w.symmetric)
    worst = 0.0
    for s in range(w.steps):
        flushes = ref.flushes
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        ref.append(tK[s], tV[s])
        assert cache.state() == (ref.Tq, ref.r)
        if ref.flushes != flushes:
            tl.assert_codes_equal(tl.gpu_packed(cache, ref.Tq), ref.packed(), w.symmetric)
        if s % check_every == 0 or s == w.steps - 1:
            out = cache.decode_attention(tl.to_dev(tQ[s], w)).cpu().numpy()
            worst = max(worst, tl.assert_close(out, ref.decode(tQ[s]), f"{w.name} step {s}"))
    return worst


@pytest.mark.parametrize("name", ALL)
def test_reduced_episode_matches_oracle(name):
    """Every workload's quantiser/geometry on a ragged prompt, every step checked,
    codes compared after prefill and after each residual flush."""
    run_episode(reduced(wl.WORKLOADS[name]))


def test_tiny_workload_exactly_as_specified():
    w = wl.WORKLOADS["tiny"]
    run_episode(w)


@pytest.mark.parametrize("limit", [1, 2, 7, 64])
def test_split_count_does_not_change_the_result(limit):
    w = reduced(wl.WORKLOADS["gqa8b"]).replace(steps=3)
    run_episode(w, split_limit=limit)


@pytest.mark.parametrize("limit", [1, 3, 64])
def test_split_count_does_not_change_the_result_mha(limit):
    # one query head per kv head: splits cut tile pairs; odd limits give uneven splits
    w = reduced(wl.WORKLOADS["llama7b"]).replace(steps=3)
    run_episode(w, split_limit=limit)


# (q heads per kv head, d, bits, G, Gv, R): every decode kernel and its ragged shapes --
# the tensor-core MHA kernel (g = 1, G >= 32), the grouped-query kernel (g = 4) and
# the CUDA-core split kernel (16-token key groups, any other g)
PATHS = [(1, 128, 4, 32, 64, 64), (1, 64, 2, 64, 16, 64), (1, 128, 2, 16, 32, 32),
         (2, 128, 2, 32, 32, 64), (8, 64, 4, 32, 32, 32), (4, 64, 4, 16, 16, 32),
         (1, 64, 4, 256, 64, 256)]


@pytest.mark.parametrize("g,d,bits,G,Gv,R", PATHS)
def test_every_decode_path(g, d, bits, G, Gv, R):
    base = wl.WORKLOADS["stream2"]
    w = base.replace(B=2, Hkv=2, Hq=2 * g, d=d, bits=bits, G=G, Gv=Gv, R=R, T=3 * R + 37,
                     steps=R + 5, k_outlier_channels=2)
    run_episode(w, check_every=7)


@pytest.mark.parametrize("name", ["llama7b", "gqa8b", "tiny", "stream4sym"])
def test_fused_append_decode_equals_separate_calls(name):
    """append_decode gives the same state, codes and (bit for bit) outputs as append followed
    by decode_attention, through flushes; and matches the oracle."""
    base = wl.WORKLOADS[name]
    w = base if name == "tiny" else reduced(base).replace(steps=base.R + 6)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    a, b = tl.new_cache(w), tl.new_cache(w)
    ref = tl.new_oracle(w)
    a.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    b.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)
    for s in range(w.steps):
        ka, va, q = tl.to_dev(tK[s], w), tl.to_dev(tV[s], w), tl.to_dev(tQ[s], w)
        a.append(ka, va)
        oa = a.decode_attention(q)
        ob = b.append_decode(ka, va, q)
        ref.append(tK[s], tV[s])
        assert a.state() == b.state() == (ref.Tq, ref.r)
        assert torch.equal(oa, ob), f"step {s}"
        if s % 9 == 0 or s == w.steps - 1:
            tl.assert_close(ob.cpu().numpy(), ref.decode(tQ[s]), f"{name} step {s}")
    Tq, r = b.state()
    tl.assert_codes_equal(tl.gpu_packed(b, Tq), ref.packed(), w.symmetric)
    assert torch.equal(a.k_residual[:, :r], b.k_residual[:, :r])
    assert torch.equal(a.v_residual[:, :r], b.v_residual[:, :r])


def test_device_status_stays_clear():
    """No bounded wait gives up in a normal decode; the status read succeeds and clears."""
    w = reduced(wl.WORKLOADS["gqa8b"]).replace(steps=2)
    XK, XV = wl.prefill_bits(w)
    _, _, tQ = wl.decode_bits(w)
    cache = tl.new_cache(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    cache.decode_attention(tl.to_dev(tQ[0], w))
    cache.check_device()
    assert kvq.load().kvq_check_device(None) == kvq.KVQ_ERR_INVALID_ARG


def test_repeated_decodes_are_identical_across_split_counts():
    """The split-merge counters return to zero after every call: the same query
    gives the same output call after call, whatever the split count in between."""
    w = reduced(wl.WORKLOADS["llama7b"]).replace(steps=1)
    XK, XV = wl.prefill_bits(w)
    _, _, tQ = wl.decode_bits(w)
    cache = tl.new_cache(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    q = tl.to_dev(tQ[0], w)
    first = cache.decode_attention(q).clone()
    for limit in (5, 1, 64, 2, 64):
        cache.set_split_limit(limit)
        out = cache.decode_attention(q)
        if limit == 64:
            assert torch.equal(out, first)
        else:
            tl.assert_close(out.cpu().numpy(), first.cpu().numpy().astype(np.float64), f"limit {limit}")


def test_prefill_then_append_equals_longer_prefill_on_gpu():
    w = reduced(wl.WORKLOADS["stream2"])
    T, k = 100, 170
    XK, XV = wl.prefill_bits(w, T=T + k)
    a = tl.new_cache(w, capacity=T + k + w.R)
    a.prefill_quantize(tl.to_dev(XK[:, :, :T], w), tl.to_dev(XV[:, :, :T], w))
    for i in range(k):
        a.append(tl.to_dev(np.ascontiguousarray(XK[:, :, T + i]), w),
                 tl.to_dev(np.ascontiguousarray(XV[:, :, T + i]), w))
    b = tl.new_cache(w, capacity=T + k + w.R)
    b.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    assert a.state() == b.state() == ((T + k) // w.R * w.R, (T + k) % w.R)
    Tq, r = a.state()
    tl.assert_codes_equal(tl.gpu_packed(a, Tq), tl.gpu_packed(b, Tq), w.symmetric)
    assert torch.equal(a.k_residual[:, :r], b.k_residual[:, :r])
    assert torch.equal(a.v_residual[:, :r], b.v_residual[:, :r])


@pytest.mark.parametrize("name", ["gqa8b", "llama7b"])
@pytest.mark.parametrize("T", [1, 15, 16, 127])
def test_all_residual_and_tiny_prompts(T, name):
    """No quantized token (T < R): plain softmax attention over the residual."""
    w = reduced(wl.WORKLOADS[name]).replace(T=T, steps=2)
    run_episode(w)


def test_empty_prompt_then_appends_through_a_flush():
    w = reduced(wl.WORKLOADS["tiny"]).replace(T=0, steps=wl.WORKLOADS["tiny"].R + 3)
    cache = tl.new_cache(w)
    ref = tl.new_oracle(w)
    tK, tV, tQ = wl.decode_bits(w)
    with pytest.raises(kvq.KVQError) as ei:
        cache.decode_attention(tl.to_dev(tQ[0], w))
    assert ei.value.status == kvq.KVQ_ERR_STATE
    for s in range(w.steps):
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        ref.append(tK[s], tV[s])
        out = cache.decode_attention(tl.to_dev(tQ[s], w)).cpu().numpy()
        tl.assert_close(out, ref.decode(tQ[s]), f"step {s}")
    tl.assert_codes_equal(tl.gpu_packed(cache, ref.Tq), ref.packed(), False)


@pytest.mark.parametrize("bits,symmetric", [(2, False), (4, False), (4, True), (2, True)])
def test_constant_and_zero_groups(bits, symmetric):
    """Constant key channels / value groups and all-zero groups: bit-exact codes."""
    w = reduced(wl.WORKLOADS["stream2"]).replace(bits=bits, symmetric=symmetric, steps=2)
    XK, XV = wl.prefill_bits(w)
    XK[:, :, :, 5] = wl.to_bits(np.float32(1.5), w.dtype)      # constant channel
    XK[:, :, :, 9] = 0                                         # zero channel
    XK[:, 1, :w.G, 20] = wl.to_bits(np.float32(-3.25), w.dtype)
    XV[:, :, 7, :] = wl.to_bits(np.float32(0.75), w.dtype)     # constant token
    XV[:, :, 8, :] = 0
    cache = tl.new_cache(w)
    ref = tl.new_oracle(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)
    tl.assert_codes_equal(tl.gpu_packed(cache, ref.Tq), ref.packed(), symmetric)
    _, _, tQ = wl.decode_bits(w)
    tl.assert_close(cache.decode_attention(tl.to_dev(tQ[0], w)).cpu().numpy(), ref.decode(tQ[0]))


def test_errors_leave_state_unchanged():
    w = reduced(wl.WORKLOADS["tiny"]).replace(T=64, steps=1)
    XK, XV = wl.prefill_bits(w)
    cache = tl.new_cache(w, capacity=64)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    st = cache.state()
    with pytest.raises(kvq.KVQError) as ei:
        cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    assert ei.value.status == kvq.KVQ_ERR_STATE and cache.state() == st
    tK, tV, tQ = wl.decode_bits(w, steps=w.R)
    for s in range(w.R - 1):
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
    st = cache.state()
    with pytest.raises(kvq.KVQError) as ei:          # this append would flush past capacity
        cache.append(tl.to_dev(tK[-1], w), tl.to_dev(tV[-1], w))
    assert ei.value.status == kvq.KVQ_ERR_CAPACITY and cache.state() == st
    q = tl.to_dev(tQ[0], w)
    ws = cache.workspace
    lib = kvq.load()
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    assert lib.kvq_decode_attention(cache._h, q.data_ptr() + 2, out.data_ptr(), ws.data_ptr(),
                                    ws.numel() * 4, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_decode_attention(cache._h, q.data_ptr(), out.data_ptr(), ws.data_ptr(),
                                    16, None) == kvq.KVQ_ERR_INVALID_ARG
    assert cache.state() == st


# ---------------------------------------------------------------------------
# full-size workloads, sampled slices
# ---------------------------------------------------------------------------

def _full_size(name, samples):
    """Run the full workload on the GPU (the launch configuration the benchmark
    times) and compare sampled (batch, kv-head) slices with the oracle run on
    those slices alone: codes after prefill and after each flush, outputs of
    the first, a middle and the last step."""
    w = wl.WORKLOADS[name]
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    cache = tl.new_cache(w)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    del XK, XV
    torch.cuda.synchronize()
    refs = {}
    for (b, h) in samples:
        xk, xv = wl.prefill_bits(w, bs=[b], hs=[h])
        o = tl.new_oracle(w, B=1, Hq=w.g, Hkv=1)
        o.prefill(xk, xv)
        refs[(b, h)] = o
        tl.assert_codes_equal(tl.gpu_packed(cache, o.Tq, bh=b * w.Hkv + h), o.packed(),
                              w.symmetric)
    check = {0, w.steps // 2, w.steps - 1}
    for s in range(w.steps):
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        out = cache.decode_attention(tl.to_dev(tQ[s], w))
        for (b, h), o in refs.items():
            fl = o.flushes
            o.append(tK[s, b:b + 1, h:h + 1], tV[s, b:b + 1, h:h + 1])
            if o.flushes != fl:
                tl.assert_codes_equal(tl.gpu_packed(cache, o.Tq, bh=b * w.Hkv + h), o.packed(),
                                      w.symmetric)
            if s in check:
                got = out[b, h * w.g:(h + 1) * w.g].cpu().numpy()
                want = o.decode(tQ[s, b:b + 1, h * w.g:(h + 1) * w.g])[0]
                tl.assert_close(got, want, f"{name} step {s} slice {(b, h)}")
    assert cache.state() == (refs[samples[0]].Tq, refs[samples[0]].r)


@pytest.mark.parametrize("name", [n for n in ALL if n != "tiny"])
def test_full_size_workload_sampled(name):
    w = wl.WORKLOADS[name]
    _full_size(name, [(0, 0), (w.B - 1, w.Hkv - 1)])


@pytest.mark.parametrize("name,world", [("llama7b", 2), ("gqa8b", 2), ("tiny", 3)])
def test_token_split_partials_merge_to_the_full_decode(name, world):
    """Shard caches of one prompt (token_split.shard_bounds; the last takes the appends):
    their partials merged by kvq_merge_partials equal the single-cache decode and the oracle."""
    from bit_kv_cache_22_b200 import token_split
    base = wl.WORKLOADS[name]
    w = base.replace(T=3 * base.R + 40, steps=9) if name == "tiny" else \
        reduced(base).replace(T=3 * base.R + 40, steps=9)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    full = tl.new_cache(w)
    full.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    shards = []
    for k, (lo, hi) in enumerate(token_split.shard_bounds(w.T, world, w.R)):
        last = k == world - 1
        cap = max(w.R, -(-((hi - lo) + (w.steps if last else 0)) // w.R) * w.R)
        c = tl.new_cache(w, capacity=cap)
        if hi > lo:
            c.prefill_quantize(tl.to_dev(np.ascontiguousarray(XK[:, :, lo:hi]), w),
                               tl.to_dev(np.ascontiguousarray(XV[:, :, lo:hi]), w))
        shards.append(c)
    ref = tl.new_oracle(w)
    ref.prefill(XK, XV)
    for s in range(w.steps):
        kk, vv, q = tl.to_dev(tK[s], w), tl.to_dev(tV[s], w), tl.to_dev(tQ[s], w)
        full.append(kk, vv)
        shards[-1].append(kk, vv)
        ref.append(tK[s], tV[s])
        parts = [c.decode_attention_partial(q) for c in shards if c.state() != (0, 0)]
        got = kvq.merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]),
                                 torch.stack([p[2] for p in parts]))
        want = full.decode_attention(q)
        torch.testing.assert_close(got, want, rtol=1e-4, atol=1e-5)
        if s % 4 == 0:
            tl.assert_close(got.cpu().numpy(), ref.decode(tQ[s]), f"{name} token split step {s}")


def test_merge_partials_of_one_and_of_an_empty_partial():
    w = reduced(wl.WORKLOADS["gqa8b"]).replace(steps=1)
    XK, XV = wl.prefill_bits(w)
    _, _, tQ = wl.decode_bits(w)
    c = tl.new_cache(w)
    c.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    q = tl.to_dev(tQ[0], w)
    o, m, l = c.decode_attention_partial(q)
    want = c.decode_attention(q)
    one = kvq.merge_partials(o[None], m[None], l[None])
    torch.testing.assert_close(one, want, rtol=1e-6, atol=1e-7)
    empty = (torch.zeros_like(o), torch.full_like(m, float("-inf")), torch.zeros_like(l))
    two = kvq.merge_partials(torch.stack([empty[0], o]), torch.stack([empty[1], m]), torch.stack([empty[2], l]))
    torch.testing.assert_close(two, want, rtol=1e-6, atol=1e-7)
