"""The GPU quantizer on the rounding and clamping edge cases, through the C ABI.

The quantizer ("Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
核心公式 / 量化基础: s = (max - min)/(2^n - 1), z = round(-min/s),
q = clamp(round(x/s) + z, 0, 2^n - 1), round half to even in fp32; symmetric int4
s = 2 max|x| / 15, q = clamp(round(x/s), -8, 7)) is fed groups built to sit on its
edges, embedded as key channels (a key group is G tokens of one channel) and as value
groups (Gv channels of one token) of a small cache:

* every hand-worked example of tests/golden/quant_hand_examples.json (ties at 0.5,
  1.5, -1.5, 13.5, a negative zero point, the clamp at 16, the symmetric 7.5 -> 8 -> 7,
  constant and all-zero groups);
* every 2-bit pattern of length 4 that uses codes 0 and 3, on grids (q - z) 2^k;
* exact ties x = (k + 1/2) s for 2-bit, 4-bit and symmetric int4;
* near-ties: the bf16 / fp16 values whose fp32 quotient x/s lies closest to a
  half-integer for scales that are not powers of two, on either side of the tie.

Codes, scales and zeros of the prefill path and of the residual-flush path must equal
the oracle's bit for bit, and the golden cases must also equal their printed values.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

import kvq_testlib as tl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "quant_hand_examples.json")))


def _rep(x, n):
    """Pad a group to n elements by repeating it (min, max and every code are unchanged)."""
    x = np.asarray(x, np.float32)
    return np.resize(x, n).astype(np.float32)


def _exact_ties(bits, symmetric):
    """Groups whose interior values are exact ties (k + 1/2) s, s a power of two."""
    out = []
    for j in (-2, 0, 3):
        s = 2.0 ** j
        if symmetric:
            # max|x| = 7.5 s gives s exactly; x/s = k + 1/2 for k = -8 .. 6
            out.append(np.array([-7.5 * s] + [(k + 0.5) * s for k in range(-8, 7)] + [7.5 * s], np.float32))
        else:
            L = (1 << bits) - 1
            for m in (0, 1, 2):                      # min = -m s: zero point m
                vals = [-m * s, (L - m) * s] + [(k + 0.5) * s for k in range(-m, L - m)]
                out.append(np.array(vals, np.float32))
    return out


def _near_ties(bits, symmetric, dtype, count=12):
    """Groups (min, max fixed; s not a power of two) holding the e-representable values
    whose fp32 quotient x/s is nearest a half-integer: the cases where a division
    shortcut would round the wrong way."""
    rng = np.random.default_rng(7 + bits + 2 * symmetric + 4 * dtype)
    out = []
    for lo, hi in ((-1.0, 1.0), (-0.3, 2.7), (0.0, 5.0), (-13.0, 0.25)):
        lo32, hi32 = np.float32(lo), np.float32(hi)
        # every e value in [lo, hi]
        grid = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
        vals = wl.from_bits(grid, dtype)
        vals = vals[np.isfinite(vals) & (vals >= lo32) & (vals <= hi32)]
        if symmetric:
            A = max(abs(lo32), abs(hi32))
            s = np.float32(np.float32(2.0) * np.float32(A)) / np.float32(15.0)
            q = (vals / s).astype(np.float32)
        else:
            s = np.float32(hi32 - lo32) / np.float32((1 << bits) - 1)
            q = (vals / s).astype(np.float32)
        dist = np.abs(q - np.floor(q) - np.float32(0.5))
        pick = vals[np.argsort(dist, kind="stable")[:count]]
        rng.shuffle(pick)
        out.append(np.concatenate([[lo32, hi32], pick]).astype(np.float32))
    return out


def _fixed_points():
    out = []
    for pattern in itertools.product(range(4), repeat=4):
        if 0 not in pattern or 3 not in pattern:
            continue
        for z, k in ((0, 0), (1, -3), (3, 2), (-5, 0)):
            out.append(np.array([(q - z) * 2.0 ** k for q in pattern], np.float32))
    return out


def _golden_cases(bits, symmetric):
    key = "symmetric" if symmetric else "asymmetric"
    return [c for c in GOLDEN[key] if c["bits"] == bits]


def _build(bits, symmetric, dtype, G, Gv, d, R):
    """Key and value inputs [1][1][T][d] holding every edge case, the rest N(0,1), and
    where each golden case sits: ('k', group, channel) or ('v', token, value group)."""
    cases = [np.array(c["x"], np.float32) for c in _golden_cases(bits, symmetric)]
    golden_n = len(cases)
    cases += _exact_ties(bits, symmetric) + _near_ties(bits, symmetric, dtype)
    if bits == 2 and not symmetric:
        cases += _fixed_points()
    # every case once as a key channel group and once as a value group
    n_kgroups = -(-len(cases) // d)
    T = -(-max(n_kgroups * G, len(cases) // (d // Gv) + 1) // R) * R
    rng = np.random.default_rng(3 + bits)
    XK = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    XV = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    where = []
    for i, x in enumerate(cases):
        g, c = divmod(i, d)
        XK[0, 0, g * G:(g + 1) * G, c] = _rep(x, G)
        t, v = divmod(i, d // Gv)
        XV[0, 0, t, v * Gv:(v + 1) * Gv] = _rep(x, Gv)
        if i < golden_n:
            where.append((("k", g, c), ("v", t, v)))
    return wl.to_bits(XK, dtype), wl.to_bits(XV, dtype), T, where


GEOMS = [  # bits, symmetric, dtype, G, Gv, d, R
    (2, False, wl.BF16, 16, 16, 64, 32),
    (4, False, wl.BF16, 32, 32, 128, 64),
    (4, True, wl.BF16, 16, 16, 64, 32),
    (2, False, wl.FP16, 32, 16, 64, 32),
    (4, False, wl.FP16, 16, 16, 64, 16),
    (4, True, wl.FP16, 32, 32, 128, 32),
    (2, False, wl.FP16, 32, 32, 128, 64),   # two key groups per CTA, batched value parameters
    (2, False, wl.BF16, 32, 32, 128, 32),   # a flush of one key group: one group per CTA
]


@pytest.mark.parametrize("bits,symmetric,dtype,G,Gv,d,R", GEOMS)
def test_quantizer_edge_cases_match_oracle_and_golden(bits, symmetric, dtype, G, Gv, d, R):
    XK, XV, T, where = _build(bits, symmetric, dtype, G, Gv, d, R)
    w = wl.WORKLOADS["tiny"].replace(B=1, Hq=1, Hkv=1, d=d, T=T, steps=0, dtype=dtype, bits=bits, G=G,
                                     Gv=Gv, R=R, symmetric=symmetric)
    ref = tl.new_oracle(w)
    ref.prefill(XK, XV)
    assert ref.Tq == T
    want = ref.packed()

    # prefill path
    a = tl.new_cache(w, capacity=T)
    a.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    got = tl.gpu_packed(a, T)
    tl.assert_codes_equal(got, want, symmetric)

    # residual-flush path: the same tokens appended one by one, quantized R at a time
    b = tl.new_cache(w, capacity=T)
    for t in range(T):
        b.append(tl.to_dev(XK[:, :, t], w), tl.to_dev(XV[:, :, t], w))
    assert b.state() == (T, 0)
    tl.assert_codes_equal(tl.gpu_packed(b, T), want, symmetric)

    # the golden cases at their places, against the printed codes, scales and zeros
    import oracle
    half = 1 << (bits - 1)
    kc = oracle.unpack(got["Kc"], T, d, bits, False)[0]     # [T][d]
    vc = oracle.unpack(got["Vc"], T, d, bits, True)[0]
    for case, (kpos, vpos) in zip(_golden_cases(bits, symmetric), where):
        n = len(case["x"])
        want_codes = case["u"] if symmetric else case["codes"]
        _, g, c = kpos
        assert kc[g * G:g * G + n, c].tolist() == want_codes, case["note"]
        assert got["Ks"][0, g, c] == np.float32(case["s"]), case["note"]
        _, t, v = vpos
        assert vc[t, v * Gv:v * Gv + n].tolist() == want_codes, case["note"]
        assert got["Vs"][0, t, v] == np.float32(case["s"]), case["note"]
        if not symmetric:
            assert got["Kz"][0, g, c] == case["z"] and got["Vz"][0, t, v] == case["z"], case["note"]
        else:
            assert all(u - half == q for u, q in zip(want_codes, case["q"]))
