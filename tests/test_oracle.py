"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: values worked by
hand from the pages' formulas (tests/golden), exact rational arithmetic,
closed-form invariants, a library attention routine, or the published
fragment table of the tensor-core operand the storage layout follows.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from bit_kv_cache_22_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# element widening against library conversions
# ---------------------------------------------------------------------------

def test_widen_fp16_every_pattern(oracle_mod):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float32)
    got = oracle_mod.widen(pats, oracle_mod.FP16)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.all(np.isinf(got[np.isinf(ref)]))


def test_widen_bf16_every_pattern(oracle_mod):
    pats = np.arange(65536, dtype=np.int32).astype(np.int16)
    ref = torch.from_numpy(pats).view(torch.bfloat16).float().numpy()
    got = oracle_mod.widen(pats.view(np.uint16), oracle_mod.BF16)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))


# ---------------------------------------------------------------------------
# hand-worked examples
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden("quant_hand_examples.json")["asymmetric"],
                         ids=lambda c: c["note"][:30])
def test_asym_hand_examples(oracle_mod, case):
    x = np.array(case["x"], np.float32)
    codes, s, z = oracle_mod.asym_codes(x, case["bits"])
    assert s == case["s"] and z == case["z"]
    assert codes.tolist() == case["codes"]
    assert [oracle_mod.dequant(q, s, z) for q in codes] == case["xdeq"]


@pytest.mark.parametrize("case", _golden("quant_hand_examples.json")["symmetric"],
                         ids=lambda c: c["note"][:30])
def test_sym_hand_examples(oracle_mod, case):
    x = np.array(case["x"], np.float32)
    u, s = oracle_mod.sym_codes(x, case["bits"])
    half = 1 << (case["bits"] - 1)
    assert s == case["s"]
    assert u.tolist() == case["u"]
    assert (u - half).tolist() == case["q"]
    assert [oracle_mod.dequant(q, s, half) for q in u] == case["xdeq"]


# ---------------------------------------------------------------------------
# invariants of the asymmetric / symmetric quantizers
# ---------------------------------------------------------------------------

def _random_groups(rng, n_groups, size):
    kinds = rng.integers(0, 4, n_groups)
    for kind in kinds:
        x = rng.standard_normal(size).astype(np.float32)
        if kind == 1:
            x = x * np.float32(rng.uniform(1e-3, 1e3))
        elif kind == 2:
            x = np.abs(x) + np.float32(rng.uniform(0, 50))      # all positive
        elif kind == 3:
            x = wl.from_bits(wl.to_bits(x * 7, wl.BF16), wl.BF16)  # bf16 grid
        yield x.astype(np.float32)


@pytest.mark.parametrize("bits", [2, 4])
def test_asym_invariants(oracle_mod, bits):
    """Codes in range; min -> 0; |x - x'| <= s/2 up to fp32 rounding."""
    rng = np.random.default_rng(11 + bits)
    L = (1 << bits) - 1
    for x in _random_groups(rng, 300, int(rng.integers(2, 64))):
        codes, s, z = oracle_mod.asym_codes(x, bits)
        assert codes.min() >= 0 and codes.max() <= L
        assert codes[np.argmin(x)] == 0
        deq = (codes.astype(np.float64) - z) * np.float64(s)
        bound = s / 2 * (1 + 2.0 ** -20) + 2.0 ** -22 * np.abs(x).max()
        assert np.all(np.abs(x.astype(np.float64) - deq) <= bound)
        # s * L reproduces the range to fp32 rounding
        assert abs(np.float64(s) * L - (np.float64(x.max()) - x.min())) <= \
            2.0 ** -22 * max(abs(x.max()), abs(x.min()), 1e-30) * 4


def test_asym_constant_group_exact(oracle_mod):
    for v in [0.0, 1.0, -1.0, 3.140625, -1e-5, 123.5, -65504.0]:
        for bits in (2, 4):
            x = np.full(8, v, np.float32)
            codes, s, z = oracle_mod.asym_codes(x, bits)
            assert np.all(codes == 0)
            assert oracle_mod.dequant(0, s, z) == np.float64(np.float32(v))


def _near_half_integer(r: Fraction, ulps: float, scale: float) -> bool:
    frac = r - math.floor(r)
    return abs(frac - Fraction(1, 2)) <= Fraction(ulps) * Fraction(scale) * Fraction(2) ** -23


@pytest.mark.parametrize("bits", [2, 4])
def test_asym_bruteforce_nearest_grid_point(oracle_mod, bits):
    """The code is the grid point (q - z) s nearest x, by exact rational search;
    z is the integer nearest -min/s."""
    rng = np.random.default_rng(5 + bits)
    L = (1 << bits) - 1
    checked = 0
    for x in _random_groups(rng, 200, 6):
        codes, s, z = oracle_mod.asym_codes(x, bits)
        S = Fraction(float(s))
        r = -Fraction(float(x.min())) / S
        if not _near_half_integer(r, 4, abs(float(r)) + 1):
            assert z == round(r)
        for xi, qi in zip(x, codes):
            X = Fraction(float(xi))
            if _near_half_integer(X / S, 4, abs(float(X / S)) + 1):
                continue
            best = min(range(L + 1), key=lambda q: abs(X - (q - z) * S))
            # (with a clamped grid of L+1 points; ties impossible off half-integers)
            assert qi == best, (xi, s, z)
            checked += 1
    assert checked > 500


def test_asym_fixed_points_every_2bit_pattern(oracle_mod):
    """A group made of grid values (q - z) 2^k that uses codes 0 and 3 reproduces
    its codes, s = 2^k and z exactly."""
    n = 0
    for pattern in itertools.product(range(4), repeat=4):
        if 0 not in pattern or 3 not in pattern:
            continue
        for z in (-5, 0, 1, 2, 3, 7):
            for k in (-3, 0, 2):
                x = np.array([(q - z) * 2.0 ** k for q in pattern], np.float32)
                codes, s, zz = oracle_mod.asym_codes(x, 2)
                assert codes.tolist() == list(pattern)
                assert s == 2.0 ** k and zz == z
                n += 1
    assert n == 6 * 3 * (256 - 2 * 81 + 16)


@pytest.mark.parametrize("bits", [2, 4])
def test_sym_invariants(oracle_mod, bits):
    rng = np.random.default_rng(21 + bits)
    half = 1 << (bits - 1)
    for x in _random_groups(rng, 300, int(rng.integers(2, 64))):
        u, s = oracle_mod.sym_codes(x, bits)
        assert u.min() >= 0 and u.max() <= 2 * half - 1
        deq = (u.astype(np.float64) - half) * np.float64(s)
        bound = s / 2 * (1 + 2.0 ** -20) + 2.0 ** -22 * np.abs(x).max()
        assert np.all(np.abs(x.astype(np.float64) - deq) <= bound)
        # symmetric grid: the scale spans [-max|x|, max|x|] in 2^n - 1 steps
        assert abs(np.float64(s) * (2 * half - 1) - 2 * np.abs(x).max()) <= \
            2.0 ** -21 * np.abs(x).max()


# ---------------------------------------------------------------------------
# packed layout
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden("layout_positions.json")["cases"],
                         ids=lambda c: f"t{c['t']}c{c['c']}v{int(c['is_v'])}d{c['d']}n{c['bits']}")
def test_layout_hand_positions(oracle_mod, case):
    w, b = oracle_mod.code_position(case["t"], case["c"], case["is_v"], case["d"], case["bits"])
    assert (w, b) == (case["word"], case["bit"])


@pytest.mark.parametrize("d,bits", [(32, 2), (64, 2), (128, 2), (64, 4), (128, 4)])
def test_layout_is_the_int8_mma_a_fragment(oracle_mod, d, bits):
    """Restates the PTX ISA table of the m16n8k32 8-bit A operand (lane l holds,
    in register a_i, byte b: row = l/4 + 8*(i%2), col = 4*(l%4) + b + 16*(i/2))
    and checks that shifting the lane's word right by n*(2*(j%B) + i%2) and
    keeping the low n bits of each byte yields that register: for keys a 16x32
    block spans chunks 2m, 2m+1 of one tile, for values tiles 2m, 2m+1 of one
    chunk."""
    B = 4 // bits
    W = d * bits // 64
    TW = d * bits // 2
    for lane in range(32):
        for i in range(4):
            for b in range(4):
                row = lane // 4 + 8 * (i % 2)
                col = 4 * (lane % 4) + b + 16 * (i // 2)
                for m in range(d // 32):
                    j = 2 * m + i // 2                 # keys: chunk of this column
                    want = (lane * W + j // B, 8 * b + bits * (2 * (j % B) + i % 2))
                    assert oracle_mod.code_position(row, 32 * m + col, False, d, bits) == want
                for j in range(d // 16):
                    tile = i // 2                      # values: tile of this column
                    want = (tile * TW + lane * W + j // B, 8 * b + bits * (2 * (j % B) + i % 2))
                    assert oracle_mod.code_position(col, 16 * j + row, True, d, bits) == want


@pytest.mark.parametrize("is_v", [False, True])
@pytest.mark.parametrize("d,bits", [(64, 2), (128, 4), (32, 4)])
def test_layout_bijection_and_roundtrip(oracle_mod, d, bits, is_v):
    T = 48
    full = np.full((2, T, d), (1 << bits) - 1, np.uint8)
    words = oracle_mod.pack(full, bits, is_v)
    assert words.shape == (2, T * d * bits // 32)
    assert np.all(words == 0xFFFFFFFF)           # every bit used
    seen = set()
    for t in range(T):
        for c in range(d):
            seen.add(oracle_mod.code_position(t, c, is_v, d, bits))
    assert len(seen) == T * d                    # no two codes share a slot
    rng = np.random.default_rng(3)
    q = rng.integers(0, 1 << bits, (3, T, d)).astype(np.uint8)
    assert np.array_equal(oracle_mod.unpack(oracle_mod.pack(q, bits, is_v), T, d, bits, is_v), q)


# ---------------------------------------------------------------------------
# block quantisation: KIVI grouping
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("symmetric", [False, True])
def test_quantize_kv_grouping(oracle_mod, symmetric):
    """Keys: one (s, z) per channel per G tokens; values: one per Gv channels per
    token (KIVI section 1); each reconstructs its original within s/2."""
    rng = np.random.default_rng(7)
    BH, T, d, G, Gv, bits = 3, 64, 64, 32, 16, 4
    xk = rng.standard_normal((BH, T, d)).astype(np.float32) * 3
    xv = rng.standard_normal((BH, T, d)).astype(np.float32)
    XK, XV = wl.to_bits(xk, wl.BF16), wl.to_bits(xv, wl.BF16)
    xk, xv = wl.from_bits(XK, wl.BF16), wl.from_bits(XV, wl.BF16)
    qc = oracle_mod.quantize_kv(XK, XV, wl.BF16, G, Gv, bits, symmetric)
    half = 1 << (bits - 1)
    for bh in range(BH):
        for g in range(T // G):
            for c in range(d):
                grp = xk[bh, g * G:(g + 1) * G, c]
                if symmetric:
                    u, s = oracle_mod.sym_codes(grp, bits)
                    z = half
                else:
                    u, s, z = oracle_mod.asym_codes(grp, bits)
                    assert qc["Kz"][bh, g, c] == z
                assert qc["Ks"][bh, g, c] == np.float32(s)
                assert np.array_equal(qc["Kq"][bh, g * G:(g + 1) * G, c], u)
                deq = (u.astype(np.float64) - z) * s
                assert np.all(np.abs(deq - grp) <= s / 2 * (1 + 2.0 ** -20) + 1e-6)
        for t in range(T):
            for j in range(d // Gv):
                grp = xv[bh, t, j * Gv:(j + 1) * Gv]
                if symmetric:
                    u, s = oracle_mod.sym_codes(grp, bits)
                else:
                    u, s, z = oracle_mod.asym_codes(grp, bits)
                    assert qc["Vz"][bh, t, j] == z
                assert qc["Vs"][bh, t, j] == np.float32(s)
                assert np.array_equal(qc["Vq"][bh, t, j * Gv:(j + 1) * Gv], u)


# ---------------------------------------------------------------------------
# streaming cache semantics
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,k", [(0, 70), (31, 40), (64, 1), (95, 33), (5, 0)])
def test_prefill_then_append_equals_longer_prefill(oracle_mod, T, k):
    w = wl.WORKLOADS["tiny"].replace(T=T + k, steps=0)
    XK, XV = wl.prefill_bits(w)
    R = w.R
    a = oracle_mod.OracleCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, R, w.bits, dtype=w.dtype)
    a.prefill(XK[:, :, :T], XV[:, :, :T])
    for i in range(k):
        a.append(XK[:, :, T + i], XV[:, :, T + i])
    b = oracle_mod.OracleCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, R, w.bits, dtype=w.dtype)
    b.prefill(XK, XV)
    assert a.Tq == b.Tq == ((T + k) // R) * R and a.r == b.r == (T + k) % R
    assert a.flushes == (T + k) // R - T // R
    for key in ("Kq", "Ks", "Kz", "Vq", "Vs", "Vz"):
        assert np.array_equal(a.quantized()[key], b.quantized()[key])
    assert np.array_equal(a.Kr[:, :a.r], b.Kr[:, :b.r])
    assert np.array_equal(a.Vr[:, :a.r], b.Vr[:, :b.r])


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _sdpa(q, k, v, g):
    """torch SDPA in fp64 with kv head i//g for query head i.
    q [B,Hq,d], k/v [B,Hkv,T,d] -> [B,Hq,d]."""
    q = torch.from_numpy(q.astype(np.float64))[:, :, None, :]
    k = torch.from_numpy(k.astype(np.float64)).repeat_interleave(g, dim=1)
    v = torch.from_numpy(v.astype(np.float64)).repeat_interleave(g, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v)[:, :, 0, :].numpy()


@pytest.mark.parametrize("Hq,Hkv,dtype", [(4, 4, wl.FP16), (8, 2, wl.BF16), (6, 3, wl.BF16)])
def test_all_residual_equals_textbook_attention(oracle_mod, Hq, Hkv, dtype):
    """With R > T no token is quantized: out = softmax(q K^T / sqrt d) V."""
    B, d, T, R = 2, 64, 37, 64
    rng = np.random.default_rng(Hq * 10 + Hkv)
    XK = wl.to_bits(rng.standard_normal((B, Hkv, T, d)) * 2, dtype)
    XV = wl.to_bits(rng.standard_normal((B, Hkv, T, d)), dtype)
    Q = wl.to_bits(rng.standard_normal((B, Hq, d)), dtype)
    c = oracle_mod.OracleCache(B, Hq, Hkv, d, 32, 32, R, 2, dtype=dtype)
    c.prefill(XK, XV)
    assert c.Tq == 0 and c.r == T
    got = c.decode(Q)
    ref = _sdpa(wl.from_bits(Q, dtype), wl.from_bits(XK, dtype), wl.from_bits(XV, dtype), Hq // Hkv)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bits,symmetric", [(2, False), (4, False), (4, True)])
def test_quantized_attention_equals_attention_on_dequantized(oracle_mod, bits, symmetric):
    """[A_g, A_r] over the quantized part plus residual equals textbook attention
    over the dequantized keys/values followed by the residual rows."""
    B, Hq, Hkv, d, G, Gv, R = 2, 4, 2, 64, 32, 16, 64
    T = 2 * R + 21
    rng = np.random.default_rng(bits + 10 * symmetric)
    XK = wl.to_bits(rng.standard_normal((B, Hkv, T, d)) * 3, wl.BF16)
    XV = wl.to_bits(rng.standard_normal((B, Hkv, T, d)), wl.BF16)
    Q = wl.to_bits(rng.standard_normal((B, Hq, d)), wl.BF16)
    c = oracle_mod.OracleCache(B, Hq, Hkv, d, G, Gv, R, bits, symmetric, wl.BF16)
    c.prefill(XK, XV)
    qc = c.quantized()
    Tq = c.Tq
    half = 1 << (bits - 1)
    kz = half if symmetric else qc["Kz"].astype(np.float64)
    vz = half if symmetric else qc["Vz"].astype(np.float64)
    ks = np.repeat(qc["Ks"].astype(np.float64), G, axis=1)
    kzz = np.repeat(kz, G, axis=1) if not symmetric else kz
    kdeq = (qc["Kq"].astype(np.float64) - kzz) * ks
    vs = np.repeat(qc["Vs"].astype(np.float64), Gv, axis=2)
    vzz = np.repeat(vz, Gv, axis=2) if not symmetric else vz
    vdeq = (qc["Vq"].astype(np.float64) - vzz) * vs
    xk = wl.from_bits(XK, wl.BF16).reshape(B * Hkv, T, d).astype(np.float64)
    xv = wl.from_bits(XV, wl.BF16).reshape(B * Hkv, T, d).astype(np.float64)
    # dequantized values reconstruct the prompt within half a step
    assert np.all(np.abs(kdeq - xk[:, :Tq]) <= ks / 2 * (1 + 2.0 ** -20) + 1e-6)
    assert np.all(np.abs(vdeq - xv[:, :Tq]) <= vs / 2 * (1 + 2.0 ** -20) + 1e-6)
    keys = np.concatenate([kdeq, xk[:, Tq:]], axis=1).reshape(B, Hkv, T, d)
    vals = np.concatenate([vdeq, xv[:, Tq:]], axis=1).reshape(B, Hkv, T, d)
    ref = _sdpa(wl.from_bits(Q, wl.BF16), keys, vals, Hq // Hkv)
    np.testing.assert_allclose(c.decode(Q), ref, rtol=1e-11, atol=1e-12)


def test_single_token_and_equal_logits(oracle_mod):
    B, Hq, Hkv, d = 1, 2, 1, 32
    rng = np.random.default_rng(0)
    XK = wl.to_bits(rng.standard_normal((B, Hkv, 1, d)), wl.BF16)
    XV = wl.to_bits(rng.standard_normal((B, Hkv, 1, d)), wl.BF16)
    Q = wl.to_bits(rng.standard_normal((B, Hq, d)), wl.BF16)
    c = oracle_mod.OracleCache(B, Hq, Hkv, d, 16, 16, 32, 2, dtype=wl.BF16)
    c.prefill(XK, XV)
    out = c.decode(Q)
    assert np.array_equal(out[0, 0], wl.from_bits(XV, wl.BF16)[0, 0, 0].astype(np.float64))
    # a zero query gives equal logits: the output is the mean of the values
    T = 64 + 9
    XK = wl.to_bits(rng.standard_normal((B, Hkv, T, d)), wl.BF16)
    XV = wl.to_bits(rng.standard_normal((B, Hkv, T, d)), wl.BF16)
    c = oracle_mod.OracleCache(B, Hq, Hkv, d, 16, 16, 32, 4, dtype=wl.BF16)
    c.prefill(XK, XV)
    zq = np.zeros((B, Hq, d), np.uint16)
    qc = c.quantized()
    vdeq = (qc["Vq"].astype(np.float64) - np.repeat(qc["Vz"], 16, axis=2)) * \
        np.repeat(qc["Vs"].astype(np.float64), 16, axis=2)
    allv = np.concatenate([vdeq[0], wl.from_bits(XV, wl.BF16)[0, 0, c.Tq:]], axis=0)
    np.testing.assert_allclose(c.decode(zq)[0, 1], allv.mean(axis=0), rtol=1e-12, atol=1e-13)


def test_token_order_does_not_matter(oracle_mod):
    """A . V = A_P . V_P (LogQuant summary, section 4): permuting the residual
    tokens leaves the output unchanged."""
    B, Hq, Hkv, d, T = 1, 4, 2, 64, 50
    rng = np.random.default_rng(9)
    XK = wl.to_bits(rng.standard_normal((B, Hkv, T, d)), wl.BF16)
    XV = wl.to_bits(rng.standard_normal((B, Hkv, T, d)), wl.BF16)
    Q = wl.to_bits(rng.standard_normal((B, Hq, d)), wl.BF16)
    perm = rng.permutation(T)
    outs = []
    for p in (np.arange(T), perm):
        c = oracle_mod.OracleCache(B, Hq, Hkv, d, 32, 32, 64, 2, dtype=wl.BF16)
        c.prefill(XK[:, :, p], XV[:, :, p])
        outs.append(c.decode(Q))
    np.testing.assert_allclose(outs[0], outs[1], rtol=1e-12, atol=1e-14)
