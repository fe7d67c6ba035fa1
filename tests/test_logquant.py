"""Pins of the LogQuant retention oracle ("Resumo Técnico: LogQuant", section 2,
Estratégia de Filtragem Baseada em Logaritmos; section 4): the retention rule on a
hand-derived trace and its invariants, prefill/append equivalence, the no-eviction
case against a textbook attention, and the whole cache against a brute-force
dequantize-then-attend written here with numpy."""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_22_b200 import workloads as wl


def run_rule(T, W):
    F, blocks = [], []
    for t in range(T):
        d = oracle.logquant_step(F, t, W)
        if d is not None:
            blocks.append(d)
    return F, blocks


def test_rule_hand_trace_w4():
    """W = 4, derived by hand from the rule: F fills to 3W = 12 tokens; its 2W = 8
    oldest are halved (the 2nd, 4th, 6th, 8th oldest leave), F is back to 8 tokens."""
    F, blocks = run_rule(12, 4)
    assert blocks == [[1, 3, 5, 7]]
    assert F == [0, 2, 4, 6, 8, 9, 10, 11]
    F, blocks = run_rule(16, 4)               # next event at 16 tokens: older part 0 2 4 6 8 9 10 11
    assert blocks == [[1, 3, 5, 7], [2, 6, 9, 11]]
    assert F == [0, 4, 8, 10, 12, 13, 14, 15]
    F, blocks = run_rule(20, 4)
    assert blocks[2] == [4, 10, 13, 15]
    assert F == [0, 8, 12, 14, 16, 17, 18, 19]
    F, _ = run_rule(11, 4)                     # one short of 3W: nothing leaves
    assert F == list(range(11))


@pytest.mark.parametrize("W", [4, 8, 32])
def test_rule_invariants(W):
    F, blocks = [], []
    for t in range(40 * W):
        d = oracle.logquant_step(F, t, W)
        if d is not None:
            blocks.append(d)
            assert len(d) == W and d == sorted(d)
        n = t + 1
        assert len(F) < 3 * W and len(F) == (n if n < 3 * W else n - W * len(blocks))
        assert len(F) >= min(n, 2 * W)
        assert F == sorted(F) and F[0] == 0                       # the first token stays
        assert F[-min(n, W):] == list(range(n - min(n, W), n))    # the newest W stay
        gaps = np.diff(F[1:])                                     # log spacing after the first token
        assert all(g & (g - 1) == 0 for g in gaps)
        assert all(np.diff(gaps) <= 0)
    every = sorted(F + [p for b in blocks for p in b])
    assert every == list(range(40 * W))                           # each token in exactly one place


def _cache(w, W):
    return oracle.LogQuantCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, W, w.bits, w.symmetric, w.dtype)


W0 = wl.WORKLOADS["stream2"].replace(B=2, Hkv=2, Hq=8, T=300, steps=70)


def test_prefill_then_appends_equals_longer_prefill():
    W = 32
    XK, XV = wl.prefill_bits(W0, T=W0.T + 40)
    a = _cache(W0, W)
    a.prefill(XK[:, :, :W0.T], XV[:, :, :W0.T])
    for t in range(W0.T, W0.T + 40):
        a.append(XK[:, :, t], XV[:, :, t])
    b = _cache(W0, W)
    b.prefill(XK, XV)
    assert a.F == b.F and a.block_positions == b.block_positions
    pa, pb = a.packed(), b.packed()
    for k in pa:
        assert np.array_equal(pa[k], pb[k])
    _, _, tQ = wl.decode_bits(W0)
    assert np.array_equal(a.decode(tQ[0]), b.decode(tQ[0]))


def _softmax_attention(q, K, V):
    """fp64 softmax(q K^T / sqrt(d)) V for q [B, Hq, d], K/V [B, Hkv, T, d] (float)."""
    B, Hq, d = q.shape
    g = Hq // K.shape[1]
    Kq = np.repeat(K, g, axis=1)
    Vq = np.repeat(V, g, axis=1)
    s = np.einsum("bhd,bhtd->bht", q, Kq) / np.sqrt(d)
    s -= s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return np.einsum("bht,bhtd->bhd", p, Vq)


def test_no_token_leaves_before_3w_tokens_textbook_attention():
    """Fewer than 3W tokens: all stay at full precision and the output is softmax attention,
    checked against torch's scaled_dot_product_attention in fp64."""
    W = 128
    XK, XV = wl.prefill_bits(W0, T=3 * W - 1)
    c = _cache(W0, W)
    c.prefill(XK, XV)
    assert c.Tq == 0 and len(c.F) == 3 * W - 1
    _, _, tQ = wl.decode_bits(W0)
    q = wl.from_bits(tQ[0], W0.dtype).astype(np.float64)
    K = wl.from_bits(XK, W0.dtype).astype(np.float64)
    V = wl.from_bits(XV, W0.dtype).astype(np.float64)
    g = W0.Hq // W0.Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None], torch.from_numpy(np.repeat(K, g, 1)),
        torch.from_numpy(np.repeat(V, g, 1)))[:, :, 0].numpy()
    np.testing.assert_allclose(c.decode(tQ[0]), ref, rtol=1e-10, atol=1e-12)


def test_cache_equals_brute_force_dequantize_then_attend():
    """[deq(blocks); F] attention written out with numpy: dequantize each quantized token
    with x' = (q - z) s (keys: per channel over groups of G tokens; values: per token over
    groups of Gv channels), append F's tokens, softmax attention in fp64."""
    W = 32
    c = _cache(W0, W)
    XK, XV = wl.prefill_bits(W0)
    c.prefill(XK, XV)
    tK, tV, tQ = wl.decode_bits(W0)
    for s in range(W0.steps):
        c.append(tK[s], tV[s])
    assert c.Tq > 0
    qc = c.quantized()
    G, Gv = W0.G, W0.Gv
    Kd = (qc["Kq"].astype(np.float64) - np.repeat(qc["Kz"], G, axis=1)) * np.repeat(qc["Ks"], G, axis=1)
    Vd = (qc["Vq"].astype(np.float64) - np.repeat(qc["Vz"], Gv, axis=2)) * np.repeat(qc["Vs"], Gv, axis=2)
    Kf = wl.from_bits(c.K[:, c.F], W0.dtype).astype(np.float64)
    Vf = wl.from_bits(c.V[:, c.F], W0.dtype).astype(np.float64)
    BH, d = W0.B * W0.Hkv, W0.d
    K = np.concatenate([Kd, Kf], axis=1).reshape(W0.B, W0.Hkv, -1, d)
    V = np.concatenate([Vd, Vf], axis=1).reshape(W0.B, W0.Hkv, -1, d)
    q = wl.from_bits(tQ[-1], W0.dtype).astype(np.float64)
    np.testing.assert_allclose(c.decode(tQ[-1]), _softmax_attention(q, K, V), rtol=1e-9, atol=1e-12)
