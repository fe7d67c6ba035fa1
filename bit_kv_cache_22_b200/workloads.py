"""Seeded synthetic workloads shared by the tests, the benchmark and the smoke check.

This module only draws random numbers and converts them to fp16/bf16 bit
patterns; it contains none of the quantisation or attention arithmetic.

Every tensor is drawn per (batch, kv-head) slice from its own
``numpy.random.Generator(PCG64(SeedSequence([seed, kind, b, h])))`` so that a
sampled slice of a full-size workload can be regenerated on its own.

The five workloads restate the configuration list this library is measured
on (shapes, dtypes, quantiser settings and value distributions):

* ``tiny``       B1, 2 heads MHA, d64, 256 tokens fp16; K,V ~ N(0,1) with 2 K
                 channels x10 per head; 2-bit asym, G=Gv=R=32; 8 decode steps
                 whose appended tokens are plain N(0,1); seed 0.
* ``llama7b``    B8, 32/32 heads, d128, 4096 tokens bf16; K ~ N(0,1) with 4
                 channels x8 per head, V ~ N(0,1); 4-bit asym, G=Gv=R=128;
                 128 decode steps.
* ``gqa8b``      B32, 32 q / 8 kv heads, d128, 8192 tokens bf16; K ~ N(0,1)
                 with 1% (=1) channel x10 per head, V ~ N(0, 0.5^2); 2-bit asym,
                 G=Gv=32, R=128; 64 decode steps.
* ``long131k``   B1, 32/8 heads, d128, 131072 tokens bf16; keys of the first 4
                 tokens x20 (sink-like), V ~ N(0,1); 2-bit asym, G=Gv=32, R=128;
                 32 decode steps.
* ``stream2`` / ``stream4sym``  B16, 32/8 heads, d128, 2048-token prefill bf16,
                 K with 4 channels x10 per head; 256 decode steps (two residual
                 flushes at R=128); 2-bit asym G=Gv=32, or symmetric int4.

A ragged batch for the paged cache (slots of different lengths, the way a
serving system batches requests) takes one of these workloads' shapes and
quantiser and draws each sequence's prompt length with ragged_lengths():

* ``ragged_gqa`` the gqa8b geometry and distributions with 32 slots whose
                 prompt lengths are uniform in [512, 15872] (mean 8192, the
                 gqa8b prompt); 64 decode steps; pages of 128 tokens.

Decode-step tokens follow the prompt's distribution (outlier channels
included, sink scaling excluded) except for ``tiny``, whose appended tokens
are plain N(0,1).  Queries are N(0,1).
"""
from __future__ import annotations

import dataclasses

import numpy as np

FP16, BF16 = 0, 1

# kinds of random streams
_K, _V, _OUTLIER, _TK, _TV, _TQ, _LEN = 0, 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int                  # prefill tokens
    steps: int              # decode steps
    dtype: int              # FP16 / BF16
    bits: int
    G: int
    Gv: int
    R: int
    symmetric: bool = False
    seed: int = 0
    k_outlier_channels: int = 0     # per kv head
    k_outlier_scale: float = 1.0
    k_sink_tokens: int = 0
    k_sink_scale: float = 1.0
    v_std: float = 1.0
    plain_decode_tokens: bool = False

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def capacity(self) -> int:
        """Token capacity of the quantized cache: ceil((T + steps) / R) * R."""
        return -(-(self.T + self.steps) // self.R) * self.R

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=2, Hkv=2, d=64, T=256, steps=8, dtype=FP16, bits=2,
                     G=32, Gv=32, R=32, seed=0, k_outlier_channels=2, k_outlier_scale=10.0,
                     plain_decode_tokens=True),
    "llama7b": Workload("llama7b", B=8, Hq=32, Hkv=32, d=128, T=4096, steps=128, dtype=BF16,
                        bits=4, G=128, Gv=128, R=128, seed=1, k_outlier_channels=4,
                        k_outlier_scale=8.0),
    "gqa8b": Workload("gqa8b", B=32, Hq=32, Hkv=8, d=128, T=8192, steps=64, dtype=BF16,
                      bits=2, G=32, Gv=32, R=128, seed=2, k_outlier_channels=1,
                      k_outlier_scale=10.0, v_std=0.5),
    "long131k": Workload("long131k", B=1, Hq=32, Hkv=8, d=128, T=131072, steps=32,
                         dtype=BF16, bits=2, G=32, Gv=32, R=128, seed=3, k_sink_tokens=4,
                         k_sink_scale=20.0),
    "stream2": Workload("stream2", B=16, Hq=32, Hkv=8, d=128, T=2048, steps=256, dtype=BF16,
                        bits=2, G=32, Gv=32, R=128, seed=4, k_outlier_channels=4,
                        k_outlier_scale=10.0),
    "stream4sym": Workload("stream4sym", B=16, Hq=32, Hkv=8, d=128, T=2048, steps=256,
                           dtype=BF16, bits=4, G=32, Gv=32, R=128, symmetric=True, seed=4,
                           k_outlier_channels=4, k_outlier_scale=10.0),
}


# ragged batches: base workload, prompt-length range and page size
RAGGED = {
    "ragged_gqa": dict(base=WORKLOADS["gqa8b"].replace(name="ragged_gqa", seed=5), lo=512, hi=15872,
                       page_tokens=128),
}


def ragged_lengths(w: Workload, lo: int, hi: int) -> list[int]:
    """Prompt length of each of the w.B sequences, uniform integers in [lo, hi]."""
    return [int(x) for x in _rng(w.seed, _LEN).integers(lo, hi + 1, size=w.B)]


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """Round fp32 values to fp16/bf16 (nearest, ties to even); return the bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == FP16:
        return x.astype(np.float16).view(np.uint16)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def from_bits(bits: np.ndarray, dtype: int) -> np.ndarray:
    """fp16/bf16 bit patterns -> fp32 (for building library-side test inputs)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == FP16:
        return bits.view(np.float16).astype(np.float32)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def outlier_channels(w: Workload, h: int) -> np.ndarray:
    """Outlier key channels of kv head h (drawn without replacement)."""
    if w.k_outlier_channels == 0:
        return np.zeros(0, np.int64)
    return np.sort(_rng(w.seed, _OUTLIER, h).choice(w.d, w.k_outlier_channels, replace=False))


def _k_scale(w: Workload, h: int, x: np.ndarray) -> np.ndarray:
    ch = outlier_channels(w, h)
    if ch.size:
        x[..., ch] *= np.float32(w.k_outlier_scale)
    return x


def prefill_slice(w: Workload, b: int, h: int, T: int | None = None):
    """fp32 prompt keys and values of one (batch, kv-head) slice: ([T, d], [T, d])."""
    T = w.T if T is None else T
    k = _rng(w.seed, _K, b, h).standard_normal((T, w.d), dtype=np.float32)
    v = _rng(w.seed, _V, b, h).standard_normal((T, w.d), dtype=np.float32)
    k = _k_scale(w, h, k)
    if w.k_sink_tokens:
        k[: w.k_sink_tokens] *= np.float32(w.k_sink_scale)
    if w.v_std != 1.0:
        v *= np.float32(w.v_std)
    return k, v


def decode_slice(w: Workload, b: int, h: int, steps: int | None = None):
    """fp32 decode-step keys and values of one slice: ([steps, d], [steps, d])."""
    steps = w.steps if steps is None else steps
    k = _rng(w.seed, _TK, b, h).standard_normal((steps, w.d), dtype=np.float32)
    v = _rng(w.seed, _TV, b, h).standard_normal((steps, w.d), dtype=np.float32)
    if not w.plain_decode_tokens:
        k = _k_scale(w, h, k)
        if w.v_std != 1.0:
            v *= np.float32(w.v_std)
    return k, v


def query_slice(w: Workload, b: int, i: int, steps: int | None = None) -> np.ndarray:
    """fp32 queries of (batch b, query head i) for every decode step: [steps, d]."""
    steps = w.steps if steps is None else steps
    return _rng(w.seed, _TQ, b, i).standard_normal((steps, w.d), dtype=np.float32)


def prefill_bits(w: Workload, bs=None, hs=None, T: int | None = None):
    """Prompt K and V bits [len(bs), len(hs), T, d] (uint16)."""
    bs = range(w.B) if bs is None else bs
    hs = range(w.Hkv) if hs is None else hs
    T = w.T if T is None else T
    XK = np.empty((len(bs), len(hs), T, w.d), np.uint16)
    XV = np.empty_like(XK)
    for ib, b in enumerate(bs):
        for ih, h in enumerate(hs):
            k, v = prefill_slice(w, b, h, T)
            XK[ib, ih] = to_bits(k, w.dtype)
            XV[ib, ih] = to_bits(v, w.dtype)
    return XK, XV


def decode_bits(w: Workload, bs=None, hs=None, steps: int | None = None):
    """Decode-step K/V bits [steps, len(bs), len(hs), d] and Q bits [steps, len(bs), g*len(hs), d].

    Query heads follow their kv head: kv head h owns query heads h*g .. h*g+g-1.
    """
    bs = range(w.B) if bs is None else bs
    hs = range(w.Hkv) if hs is None else hs
    steps = w.steps if steps is None else steps
    g = w.g
    tK = np.empty((steps, len(bs), len(hs), w.d), np.uint16)
    tV = np.empty_like(tK)
    tQ = np.empty((steps, len(bs), len(hs) * g, w.d), np.uint16)
    for ib, b in enumerate(bs):
        for ih, h in enumerate(hs):
            k, v = decode_slice(w, b, h, steps)
            tK[:, ib, ih] = to_bits(k, w.dtype)
            tV[:, ib, ih] = to_bits(v, w.dtype)
            for j in range(g):
                tQ[:, ib, ih * g + j] = to_bits(query_slice(w, b, h * g + j, steps), w.dtype)
    return tK, tV, tQ
