"""Pins of the dense-and-sparse key oracle (KVQuant's per-vector dense-and-sparse
quantization and SqueezeLLM's W = D + S on the "LLM系列：KVCache量化…" pages): the
outlier choice on a hand example, exact reconstruction of the outliers, the dense
part's narrower ranges and error bound, the n_out = 0 reduction to KIVI, and the
numpy attention against the C oracle's."""
import numpy as np
import pytest

import oracle
from bit_kv_cache_22_b200 import workloads as wl

W0 = wl.WORKLOADS["stream2"].replace(B=2, Hkv=2, Hq=8, T=3 * 128 + 40, steps=20)


def _bits(vals, dtype=wl.BF16):
    return wl.to_bits(np.asarray(vals, np.float32), dtype)


def test_outlier_choice_hand_example():
    # one token, 8 channels: |-5| and |5| tie, the lower channel (1) goes first; then 5 (3)
    x = _bits([[[1.0, -5.0, 3.0, 5.0, 0.5, -4.0, 2.0, 0.0]]])
    idx, vals, dense = oracle.key_outliers(x, 2, wl.BF16)
    assert idx.tolist() == [[[1, 3]]]
    assert vals.tolist() == x[..., [1, 3]].tolist()
    assert wl.from_bits(dense, wl.BF16).tolist() == [[[1.0, 0.0, 3.0, 0.0, 0.5, -4.0, 2.0, 0.0]]]
    q = oracle.quantize_kv_sparse(np.repeat(x, 16, axis=1), np.repeat(x, 16, axis=1), wl.BF16, 16, 8, 2,
                                  n_out=2)
    assert (q["Ko"][0, 0] == [(1 << 16) | int(x[0, 0, 1]), (3 << 16) | int(x[0, 0, 3])]).all()


@pytest.mark.parametrize("symmetric,bits", [(False, 2), (False, 4), (True, 4)])
def test_outliers_reconstruct_exactly_and_the_dense_part_is_narrower(symmetric, bits):
    w = W0.replace(bits=bits, symmetric=symmetric)
    XK, XV = wl.prefill_bits(w)
    XK = XK.reshape(w.B * w.Hkv, w.T, w.d)[:, :256]
    XV = XV.reshape(w.B * w.Hkv, w.T, w.d)[:, :256]
    n_out = 2
    plain = oracle.quantize_kv(XK, XV, w.dtype, w.G, w.Gv, bits, symmetric)
    sp = oracle.quantize_kv_sparse(XK, XV, w.dtype, w.G, w.Gv, bits, symmetric, n_out)
    K, _ = oracle.dequantize(sp, w.G, w.Gv, bits, symmetric, w.dtype)
    x = oracle.widen_array(XK, w.dtype)
    ch = (sp["Ko"] >> 16).astype(np.int64)
    # outliers: exact
    assert np.array_equal(np.take_along_axis(K, ch, -1), np.take_along_axis(x, ch, -1))
    # the dense part: per (group, channel) scale no larger than the plain one, and every
    # other element within half its (dense) step
    assert (sp["Ks"] <= plain["Ks"]).all()
    step = np.repeat(sp["Ks"].astype(np.float64), w.G, axis=1)
    mask = np.ones_like(x, bool)
    np.put_along_axis(mask, ch, False, axis=-1)
    err = np.abs(K - x)[mask]
    assert (err <= step[mask] / 2 * (1 + 2 ** -20) + 2 ** -22 * np.abs(x).max()).all()
    # values are untouched
    assert np.array_equal(sp["Vq"], plain["Vq"]) and np.array_equal(sp["Vs"], plain["Vs"])


def test_no_outliers_is_kivi_and_numpy_attention_matches_the_c_oracle():
    XK, XV = wl.prefill_bits(W0)
    tK, tV, tQ = wl.decode_bits(W0)
    a = oracle.SparseKeyCache(W0.B, W0.Hq, W0.Hkv, W0.d, W0.G, W0.Gv, W0.R, W0.bits, False, W0.dtype, n_out=0)
    b = oracle.OracleCache(W0.B, W0.Hq, W0.Hkv, W0.d, W0.G, W0.Gv, W0.R, W0.bits, False, W0.dtype)
    for c in (a, b):
        c.prefill(XK, XV)
        for s in range(W0.steps):
            c.append(tK[s], tV[s])
    pa, pb = a.packed(), b.packed()
    for k in pb:
        assert np.array_equal(pa[k], pb[k])
    np.testing.assert_allclose(a.decode(tQ[-1]), b.decode(tQ[-1]), rtol=1e-10, atol=1e-13)


def test_sparse_cache_equals_attention_over_the_reconstruction():
    """With outliers: attention over [deq(D) + S; residual] built independently of the class."""
    XK, XV = wl.prefill_bits(W0)
    _, _, tQ = wl.decode_bits(W0)
    c = oracle.SparseKeyCache(W0.B, W0.Hq, W0.Hkv, W0.d, W0.G, W0.Gv, W0.R, W0.bits, False, W0.dtype, n_out=1)
    c.prefill(XK, XV)
    Tq = c.Tq
    BH = W0.B * W0.Hkv
    xk = XK.reshape(BH, W0.T, W0.d)
    xv = XV.reshape(BH, W0.T, W0.d)
    # reconstruction: the plain quantiser on the dense keys, outliers put back by value
    idx, vals, dense = oracle.key_outliers(xk[:, :Tq], 1, W0.dtype)
    q = oracle.quantize_kv(dense, xv[:, :Tq], W0.dtype, W0.G, W0.Gv, W0.bits)
    Kd, Vd = oracle.dequantize(q, W0.G, W0.Gv, W0.bits, False, W0.dtype)
    np.put_along_axis(Kd, idx, oracle.widen_array(vals, W0.dtype), axis=-1)
    K = np.concatenate([Kd, oracle.widen_array(xk[:, Tq:], W0.dtype)], axis=1)
    V = np.concatenate([Vd, oracle.widen_array(xv[:, Tq:], W0.dtype)], axis=1)
    np.testing.assert_allclose(c.decode(tQ[0]), oracle.attend(K, V, tQ[0], W0.dtype, W0.B, W0.Hq, W0.Hkv),
                               rtol=1e-12, atol=1e-14)
