"""GPU parity of dense-and-sparse keys (KVQuant's per-vector dense-and-sparse
quantization, SqueezeLLM's W = D + S): codes, scales, zeros and the outlier words
bit-exact against the oracle; outputs |gpu - ref| <= 2e-3 + 1e-2 |ref|."""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

import kvq_testlib as tl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def new_sparse(w, n_out, capacity=None, window=None):
    return kvq.KVQCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, tl.torch_dtype(w),
                        capacity or w.capacity, "cuda", window=window, key_outliers=n_out)


def gpu_outliers(cache, Tq):
    return cache.k_outliers[:, :Tq].cpu().numpy().view(np.uint32)


# the tensor-core kernel with 1, 2 and 4 query heads per kv head, 2- and 4-bit, symmetric, fp16 / d64
CASES = [
    ("llama7b", dict(B=2, Hq=2, Hkv=2, T=2 * 128 + 40, steps=140), 1),
    ("gqa8b", dict(B=2, Hq=8, Hkv=2, T=2 * 128 + 40, steps=140), 2),
    ("gqa8b", dict(B=2, Hq=4, Hkv=2, T=2 * 128 + 40, steps=140, Gv=64), 1),
    ("stream4sym", dict(B=2, Hq=8, Hkv=2, T=2 * 128 + 40, steps=140), 1),
    ("tiny", dict(steps=40), 2),
]


@pytest.mark.parametrize("name,changes,n_out", CASES)
def test_sparse_keys_episode_matches_oracle(name, changes, n_out):
    w = wl.WORKLOADS[name].replace(**changes)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    cache = new_sparse(w, n_out)
    ref = oracle.SparseKeyCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, w.dtype, n_out)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)

    def codes():
        assert cache.state() == (ref.Tq, ref.r)
        tl.assert_codes_equal(tl.gpu_packed(cache, ref.Tq), ref.packed(), w.symmetric)
        assert np.array_equal(gpu_outliers(cache, ref.Tq), ref.packed()["Ko"])

    codes()
    for s in range(w.steps):
        flushes = ref.flushes
        out = cache.append_decode(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w), tl.to_dev(tQ[s], w))
        ref.append(tK[s], tV[s])
        if ref.flushes != flushes:
            codes()
        if s % 7 == 0 or s == w.steps - 1:
            tl.assert_close(out.cpu().numpy(), ref.decode(tQ[s]), f"{name} n_out={n_out} step {s}")
    cache.check_device()


def test_sparse_keys_with_logquant_retention():
    """The outliers also apply to LogQuant's quantized blocks."""
    w = wl.WORKLOADS["gqa8b"].replace(B=2, Hq=8, Hkv=2, T=300, steps=70)
    W = 32
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    cache = new_sparse(w, 1, capacity=-(-(w.T + w.steps) // W) * W, window=W)
    ref = oracle.LogQuantCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, W, w.bits, w.symmetric, w.dtype)
    cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    ref.prefill(XK, XV)
    for s in range(w.steps):
        cache.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        ref.append(tK[s], tV[s])
    # the oracle's blocks, re-quantized dense-and-sparse from the same leaving tokens
    blocks = [oracle.quantize_kv_sparse(ref.K[:, p], ref.V[:, p], w.dtype, w.G, w.Gv, w.bits, w.symmetric, 1)
              for p in ref.block_positions]
    qc = {k: np.concatenate([b[k] for b in blocks], axis=1) for k in blocks[0]}
    Tq = ref.Tq
    assert cache.state() == (Tq, len(ref.F))
    want = dict(Kc=oracle.pack(qc["Kq"], w.bits, False), Vc=oracle.pack(qc["Vq"], w.bits, True),
                Ks=qc["Ks"], Kz=qc["Kz"], Vs=qc["Vs"], Vz=qc["Vz"])
    tl.assert_codes_equal(tl.gpu_packed(cache, Tq), want, w.symmetric)
    assert np.array_equal(gpu_outliers(cache, Tq), qc["Ko"])
    Kd, Vd = oracle.dequantize(qc, w.G, w.Gv, w.bits, w.symmetric, w.dtype)
    K = np.concatenate([Kd, oracle.widen_array(ref.K[:, ref.F], w.dtype)], axis=1)
    V = np.concatenate([Vd, oracle.widen_array(ref.V[:, ref.F], w.dtype)], axis=1)
    out = cache.decode_attention(tl.to_dev(tQ[-1], w)).cpu().numpy()
    tl.assert_close(out, oracle.attend(K, V, tQ[-1], w.dtype, w.B, w.Hq, w.Hkv), "logquant + sparse")


def test_sparse_keys_errors():
    w = wl.WORKLOADS["stream2"].replace(B=1, Hq=4, Hkv=2, G=16, Gv=16, T=64)
    with pytest.raises(kvq.KVQError):
        new_sparse(w, 1)                                   # 16-token groups: the CUDA-core path
    w = wl.WORKLOADS["gqa8b"].replace(B=1, Hq=8, Hkv=2, T=200)
    c = tl.new_cache(w)
    small = torch.empty(4, dtype=torch.int32, device="cuda")
    assert c._lib.kvq_set_key_outliers(c._h, 1, small.data_ptr(), 16) == kvq.KVQ_ERR_INVALID_ARG   # too small
    XK, XV = wl.prefill_bits(w)
    c.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    buf = torch.empty(w.B * w.Hkv * w.capacity, dtype=torch.int32, device="cuda")
    assert c._lib.kvq_set_key_outliers(c._h, 1, buf.data_ptr(), buf.numel() * 4) == kvq.KVQ_ERR_STATE
