"""CPU oracle for KIVI-style low-bit KV-cache decode attention -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may use
this package.  It is a plain restatement of the method written from the
pages (see ``kvq_oracle.c`` for the passages followed): the numeric core is
plain C compiled with gcc (fp32 codes without FMA contraction or fast-math,
fp64 attention), and this module only marshals numpy arrays into it and keeps
the streaming bookkeeping of the KIVI residual (section 1 of "LLM系列：
KVCache量化1 KIVI ...": new tokens go to the full-precision residual; when it
holds R tokens it is quantized, appended to the quantized part and reset).
It also restates, each in a section of its own below with its sources: the
merge of token-split partials, LogQuant's full-precision retention
(LogQuantCache) and dense-and-sparse keys (SparseKeyCache).

It shares no code with the CUDA library and imports nothing from it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, EINVAL, ERANGE = 0, 1, 2
FP16, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (gcc, OpenMP when available)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    base = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", "-Wall"]
    tmp = _LIB + f".tmp{os.getpid()}"
    try:
        subprocess.run(base + ["-fopenmp", "-o", tmp, _SRC, "-lm"], check=True,
                       capture_output=True)
    except subprocess.CalledProcessError:
        subprocess.run(base + ["-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int
        lib.oracle_widen.restype = ctypes.c_float
        lib.oracle_widen.argtypes = [ctypes.c_uint16, i32]
        lib.oracle_asym_params.restype = i32
        lib.oracle_asym_params.argtypes = [P, i64, i64, i32, P, P]
        lib.oracle_asym_code.restype = i32
        lib.oracle_asym_code.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_int32, i32]
        lib.oracle_sym_params.restype = i32
        lib.oracle_sym_params.argtypes = [P, i64, i64, i32, P]
        lib.oracle_sym_code.restype = i32
        lib.oracle_sym_code.argtypes = [ctypes.c_float, ctypes.c_float, i32]
        lib.oracle_quantize_kv.restype = i32
        lib.oracle_quantize_kv.argtypes = [P, P, i32, i64, i64, i32, i32, i32, i32, i32,
                                           P, P, P, P, P, P]
        lib.oracle_code_position.restype = None
        lib.oracle_code_position.argtypes = [i64, i32, i32, i32, i32, P, P]
        lib.oracle_pack.restype = i32
        lib.oracle_pack.argtypes = [P, i64, i64, i32, i32, i32, P]
        lib.oracle_unpack.restype = i32
        lib.oracle_unpack.argtypes = [P, i64, i64, i32, i32, i32, P]
        lib.oracle_dequant.restype = ctypes.c_double
        lib.oracle_dequant.argtypes = [i32, ctypes.c_float, ctypes.c_int32]
        lib.oracle_decode_attention.restype = i32
        lib.oracle_decode_attention.argtypes = [P, P, P, P, P, P, i64, P, P, i64, i64, P,
                                                i32, i64, i32, i32, i32, i32, i32, i32, i32, P, P, P]
        lib.oracle_num_threads.restype = i32
        lib.oracle_num_threads.argtypes = []
        lib.oracle_set_num_threads.restype = i32
        lib.oracle_set_num_threads.argtypes = [i32]
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != OK:
        raise ValueError(f"oracle {what} rejected its input (status {rc})")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> int:
    """Threads the oracle's parallel sections use from now on; returns the previous count.
    Results do not depend on it (every parallel section writes disjoint outputs)."""
    return int(_load().oracle_set_num_threads(int(n)))


# ----------------------------------------------------------------------------
# scalar / small helpers
# ----------------------------------------------------------------------------

def widen(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Exact fp16/bf16 -> fp32 widening of an array of element bit patterns."""
    lib = _load()
    flat = np.ascontiguousarray(bits, dtype=np.uint16).ravel()
    out = np.array([lib.oracle_widen(int(b), dtype) for b in flat], dtype=np.float32)
    return out.reshape(np.shape(bits))


def asym_params(x: np.ndarray, bits: int):
    """(s, z) of one asymmetric min-max group."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.zeros(1, np.float32)
    z = np.zeros(1, np.int32)
    _check(lib.oracle_asym_params(_ptr(x), x.size, 1, bits, _ptr(s), _ptr(z)), "asym_params")
    return float(s[0]), int(z[0])


def asym_codes(x: np.ndarray, bits: int):
    """(codes, s, z) of one asymmetric group."""
    lib = _load()
    s, z = asym_params(x, bits)
    codes = np.array([lib.oracle_asym_code(float(v), s, z, bits)
                      for v in np.asarray(x, np.float32)], dtype=np.int32)
    return codes, s, z


def sym_codes(x: np.ndarray, bits: int):
    """(offset codes u, s) of one symmetric group."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.zeros(1, np.float32)
    _check(lib.oracle_sym_params(_ptr(x), x.size, 1, bits, _ptr(s)), "sym_params")
    codes = np.array([lib.oracle_sym_code(float(v), float(s[0]), bits) for v in x],
                     dtype=np.int32)
    return codes, float(s[0])


def dequant(code: int, s: float, z: int) -> float:
    return float(_load().oracle_dequant(int(code), float(s), int(z)))


def code_position(t: int, c: int, is_v: bool, d: int, bits: int):
    lib = _load()
    w = ctypes.c_int64()
    b = ctypes.c_int()
    lib.oracle_code_position(t, c, int(is_v), d, bits, ctypes.byref(w), ctypes.byref(b))
    return int(w.value), int(b.value)


# ----------------------------------------------------------------------------
# block quantisation, packing, attention
# ----------------------------------------------------------------------------

def quantize_kv(XK: np.ndarray, XV: np.ndarray, dtype: int, G: int, Gv: int, bits: int,
                symmetric: bool = False) -> dict:
    """Quantise K/V element bits shaped [BH, T, d] (KIVI: K per channel, V per token)."""
    lib = _load()
    XK = np.ascontiguousarray(XK, dtype=np.uint16)
    XV = np.ascontiguousarray(XV, dtype=np.uint16)
    BH, T, d = XK.shape
    assert XV.shape == XK.shape
    Kq = np.zeros((BH, T, d), np.uint8)
    Vq = np.zeros((BH, T, d), np.uint8)
    Ks = np.zeros((BH, T // G, d), np.float32)
    Kz = np.zeros((BH, T // G, d), np.int16)
    Vs = np.zeros((BH, T, d // Gv), np.float32)
    Vz = np.zeros((BH, T, d // Gv), np.int16)
    rc = lib.oracle_quantize_kv(_ptr(XK), _ptr(XV), dtype, BH, T, d, G, Gv, bits, int(symmetric),
                                _ptr(Kq), _ptr(Ks), _ptr(Kz), _ptr(Vq), _ptr(Vs), _ptr(Vz))
    _check(rc, "quantize_kv")
    return dict(Kq=Kq, Ks=Ks, Kz=Kz, Vq=Vq, Vs=Vs, Vz=Vz)


def pack(q: np.ndarray, bits: int, is_v: bool) -> np.ndarray:
    """Pack codes [BH, T, d] into the tile layout -> uint32 [BH, T*d*bits/32]."""
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.uint8)
    BH, T, d = q.shape
    out = np.zeros((BH, T * d * bits // 32), np.uint32)
    _check(lib.oracle_pack(_ptr(q), BH, T, d, bits, int(is_v), _ptr(out)), "pack")
    return out


def unpack(words: np.ndarray, T: int, d: int, bits: int, is_v: bool) -> np.ndarray:
    lib = _load()
    words = np.ascontiguousarray(words, dtype=np.uint32)
    BH = words.shape[0]
    q = np.zeros((BH, T, d), np.uint8)
    _check(lib.oracle_unpack(_ptr(words), BH, T, d, bits, int(is_v), _ptr(q)), "unpack")
    return q


def decode_attention(qcache: dict, Tq: int, Kr: np.ndarray, Vr: np.ndarray, r: int,
                     Q: np.ndarray, dtype: int, B: int, Hq: int, Hkv: int, d: int,
                     G: int, Gv: int, bits: int, symmetric: bool, stats: bool = False):
    """fp64 decode attention of queries Q [B, Hq, d] over [deq(quantized); residual].

    With stats=True also returns the softmax statistics (m, l) [B, Hq]: m the
    largest scaled logit, l = sum_t exp(logit_t - m)."""
    lib = _load()
    Q = np.ascontiguousarray(Q, dtype=np.uint16)
    Kr = np.ascontiguousarray(Kr, dtype=np.uint16)
    Vr = np.ascontiguousarray(Vr, dtype=np.uint16)
    Rcap = Kr.shape[1]
    out = np.zeros((B, Hq, d), np.float64)
    m = np.zeros((B, Hq), np.float64)
    l = np.zeros((B, Hq), np.float64)
    arrs = [np.ascontiguousarray(qcache[k]) for k in ("Kq", "Ks", "Kz", "Vq", "Vs", "Vz")]
    rc = lib.oracle_decode_attention(*[_ptr(a) for a in arrs], Tq, _ptr(Kr), _ptr(Vr), Rcap, r,
                                     _ptr(Q), dtype, B, Hq, Hkv, d, G, Gv, bits,
                                     int(symmetric), _ptr(out), _ptr(m), _ptr(l))
    _check(rc, "decode_attention")
    return (out, m, l) if stats else out


def merge_partials(outs, ms, ls) -> np.ndarray:
    """Output over the union of disjoint token sets from each set's (normalised) output and
    softmax statistics: sum_k w_k out_k / sum_k w_k with w_k = l_k exp(m_k - M), M = max_k m_k
    (log-sum-exp; the token order of a concatenation does not matter, LogQuant summary,
    section 4)."""
    ms = np.stack(ms)
    M = ms.max(axis=0)
    w = np.stack(ls) * np.exp(ms - M)
    num = sum(w[k][..., None] * outs[k] for k in range(len(outs)))
    return num / w.sum(axis=0)[..., None]


# ----------------------------------------------------------------------------
# streaming cache (KIVI section 1: quantized part + residual of < R tokens)
# ----------------------------------------------------------------------------

class OracleCache:
    """Prefill / append / decode with KIVI's residual.

    Prefill of T tokens quantises the first floor(T/R)*R of them and keeps the
    rest in the residual; each append adds one token to the residual and, when
    the residual reaches R tokens, quantises all R of them, appends them to
    the quantized part and empties the residual.  Attention therefore always
    sees fewer than R residual tokens.
    """

    def __init__(self, B, Hq, Hkv, d, G, Gv, R, bits, symmetric=False, dtype=BF16):
        assert R % G == 0 and d % Gv == 0 and Hq % Hkv == 0
        self.B, self.Hq, self.Hkv, self.d = B, Hq, Hkv, d
        self.G, self.Gv, self.R, self.bits = G, Gv, R, bits
        self.symmetric, self.dtype = symmetric, dtype
        BH = B * Hkv
        self.blocks = []                       # quantized blocks, each R*k tokens
        self.Kr = np.zeros((BH, R, d), np.uint16)
        self.Vr = np.zeros((BH, R, d), np.uint16)
        self.r = 0
        self.Tq = 0
        self.flushes = 0
        self._cat = None

    def _quantize_block(self, XK, XV):
        blk = quantize_kv(XK, XV, self.dtype, self.G, self.Gv, self.bits, self.symmetric)
        self.blocks.append(blk)
        self.Tq += XK.shape[1]
        self._cat = None

    def prefill(self, XK: np.ndarray, XV: np.ndarray):
        """XK, XV element bits [B, Hkv, T, d]."""
        assert self.Tq == 0 and self.r == 0
        B, Hkv, T, d = XK.shape
        XK = XK.reshape(B * Hkv, T, d)
        XV = XV.reshape(B * Hkv, T, d)
        Tq = (T // self.R) * self.R
        if Tq:
            self._quantize_block(XK[:, :Tq], XV[:, :Tq])
        self.r = T - Tq
        self.Kr[:, :self.r] = XK[:, Tq:]
        self.Vr[:, :self.r] = XV[:, Tq:]

    def append(self, tK: np.ndarray, tV: np.ndarray):
        """tK, tV element bits [B, Hkv, d]; flushes the residual when it fills."""
        BH = self.B * self.Hkv
        self.Kr[:, self.r] = tK.reshape(BH, self.d)
        self.Vr[:, self.r] = tV.reshape(BH, self.d)
        self.r += 1
        if self.r == self.R:
            self._quantize_block(self.Kr.copy(), self.Vr.copy())
            self.flushes += 1
            self.r = 0

    def quantized(self) -> dict:
        """All quantized tokens so far, concatenated along the token axis."""
        if self._cat is None:
            if not self.blocks:
                BH, d = self.B * self.Hkv, self.d
                self._cat = dict(Kq=np.zeros((BH, 0, d), np.uint8),
                                 Ks=np.zeros((BH, 0, d), np.float32),
                                 Kz=np.zeros((BH, 0, d), np.int16),
                                 Vq=np.zeros((BH, 0, d), np.uint8),
                                 Vs=np.zeros((BH, 0, d // self.Gv), np.float32),
                                 Vz=np.zeros((BH, 0, d // self.Gv), np.int16))
            else:
                self._cat = {k: np.concatenate([b[k] for b in self.blocks], axis=1)
                             for k in self.blocks[0]}
        return self._cat

    def packed(self) -> dict:
        """Quantized part in the library's storage format (codes packed)."""
        qc = self.quantized()
        return dict(Kc=pack(qc["Kq"], self.bits, False), Vc=pack(qc["Vq"], self.bits, True),
                    Ks=qc["Ks"], Kz=qc["Kz"], Vs=qc["Vs"], Vz=qc["Vz"])

    def decode(self, Q: np.ndarray, stats: bool = False):
        """Q element bits [B, Hq, d] -> fp64 output [B, Hq, d] (and (m, l) with stats=True)."""
        return decode_attention(self.quantized(), self.Tq, self.Kr, self.Vr, self.r, Q,
                                self.dtype, self.B, self.Hq, self.Hkv, self.d, self.G,
                                self.Gv, self.bits, self.symmetric, stats)


# ----------------------------------------------------------------------------
# LogQuant retention ("Resumo Técnico: LogQuant", section 2, Estratégia de
# Filtragem Baseada em Logaritmos, and section 4): which tokens stay in full
# precision.  Reading taken (the summary is terse): the full-precision set F
# holds at most 3W tokens (the 3W reserve); every new token enters F; when F
# reaches 3W tokens, the density of its older part is halved -- of its 2W oldest
# tokens every other one (the 2nd, 4th, ... oldest) leaves F -- which brings the
# older part from 2W to W tokens before new tokens fill F up again.  The W
# tokens that leave are quantized together as one block (KIVI's quantiser,
# groups of G tokens inside the block), appended to the quantized part in the
# order the blocks leave.  Attention runs over [dequantized blocks; F]: the
# order of a concatenation does not change it (section 4).  Repeated halving
# leaves F log-spaced: the newest tokens dense, older ones at strides 2, 4, ...
# ----------------------------------------------------------------------------

def logquant_step(F: list, t: int, W: int):
    """Token position t enters F (ascending positions).  Returns the block of W
    positions that leaves F (ascending), or None."""
    F.append(t)
    if len(F) < 3 * W:
        return None
    older = F[:2 * W]
    dropped = older[1::2]
    F[:] = older[0::2] + F[2 * W:]
    return dropped


class LogQuantCache:
    """Prefill / append / decode with LogQuant's full-precision retention and
    KIVI's quantiser for the tokens that leave it.  Element bits as in OracleCache;
    every token is kept here at full precision too, to quantize it when it leaves."""

    def __init__(self, B, Hq, Hkv, d, G, Gv, W, bits, symmetric=False, dtype=BF16):
        assert W % G == 0 and d % Gv == 0 and Hq % Hkv == 0
        self.B, self.Hq, self.Hkv, self.d = B, Hq, Hkv, d
        self.G, self.Gv, self.W, self.bits = G, Gv, W, bits
        self.symmetric, self.dtype = symmetric, dtype
        BH = B * Hkv
        self.K = np.zeros((BH, 64, d), np.uint16)     # every token so far, by position
        self.V = np.zeros((BH, 64, d), np.uint16)
        self.n = 0
        self.F = []                                  # full-precision positions
        self.block_positions = []                    # positions of each quantized block
        self.blocks = []
        self.Tq = 0

    def _push(self, k: np.ndarray, v: np.ndarray):
        if self.n == self.K.shape[1]:
            self.K = np.concatenate([self.K, np.zeros_like(self.K)], axis=1)
            self.V = np.concatenate([self.V, np.zeros_like(self.V)], axis=1)
        self.K[:, self.n] = k
        self.V[:, self.n] = v
        dropped = logquant_step(self.F, self.n, self.W)
        self.n += 1
        if dropped is not None:
            self.block_positions.append(dropped)
            self.blocks.append(quantize_kv(self.K[:, dropped], self.V[:, dropped], self.dtype,
                                           self.G, self.Gv, self.bits, self.symmetric))
            self.Tq += self.W

    def prefill(self, XK: np.ndarray, XV: np.ndarray):
        """XK, XV element bits [B, Hkv, T, d]: the tokens enter one by one."""
        assert self.n == 0
        B, Hkv, T, d = XK.shape
        XK = XK.reshape(B * Hkv, T, d)
        XV = XV.reshape(B * Hkv, T, d)
        for t in range(T):
            self._push(XK[:, t], XV[:, t])

    def append(self, tK: np.ndarray, tV: np.ndarray):
        BH = self.B * self.Hkv
        self._push(tK.reshape(BH, self.d), tV.reshape(BH, self.d))

    def quantized(self) -> dict:
        if not self.blocks:
            BH, d = self.B * self.Hkv, self.d
            return dict(Kq=np.zeros((BH, 0, d), np.uint8), Ks=np.zeros((BH, 0, d), np.float32),
                        Kz=np.zeros((BH, 0, d), np.int16), Vq=np.zeros((BH, 0, d), np.uint8),
                        Vs=np.zeros((BH, 0, d // self.Gv), np.float32),
                        Vz=np.zeros((BH, 0, d // self.Gv), np.int16))
        return {k: np.concatenate([b[k] for b in self.blocks], axis=1) for k in self.blocks[0]}

    def packed(self) -> dict:
        qc = self.quantized()
        return dict(Kc=pack(qc["Kq"], self.bits, False), Vc=pack(qc["Vq"], self.bits, True),
                    Ks=qc["Ks"], Kz=qc["Kz"], Vs=qc["Vs"], Vz=qc["Vz"])

    def decode(self, Q: np.ndarray, stats: bool = False):
        """Q element bits [B, Hq, d] -> fp64 output over [deq(blocks); F]."""
        Kr = np.ascontiguousarray(self.K[:, self.F])
        Vr = np.ascontiguousarray(self.V[:, self.F])
        return decode_attention(self.quantized(), self.Tq, Kr, Vr, len(self.F), Q, self.dtype,
                                self.B, self.Hq, self.Hkv, self.d, self.G, self.Gv, self.bits,
                                self.symmetric, stats)


# ----------------------------------------------------------------------------
# Dense-and-sparse keys ("LLM系列：KVCache量化…" pages: KVQuant, point (4)
# Per-Vector Dense-and-Sparse Quantization -- a small share of outliers, e.g.
# 1%, is kept at full precision in a separate sparse matrix; SqueezeLLM,
# section (2) Dense-and-Sparse decomposition W = D + S, WX = DX + SX).
# Reading taken: the vector is one token's key (d channels of one kv head); its
# n_out entries of largest magnitude (ties: the lower channel first) form the
# sparse part S and are set to +0 in the dense part D, which KIVI's quantiser
# then quantizes as usual.  Since D holds that 0, every group that contains it
# has min <= 0 <= max and quantizes the 0 to code z, which dequantizes to
# exactly 0; so deq(D) + S is exact at the outliers.  Values are unchanged.
# ----------------------------------------------------------------------------

def widen_array(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Exact fp16/bf16 -> fp64 widening of a whole array (bf16: the bits are the high half of
    an fp32; fp16 through numpy's half type)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == FP16:
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def key_outliers(XK: np.ndarray, n_out: int, dtype: int):
    """XK element bits [BH, T, d] -> (channels [BH, T, n_out], their bits, dense bits)."""
    XK = np.ascontiguousarray(XK, dtype=np.uint16)
    mag = np.abs(widen_array(XK, dtype))
    order = np.argsort(-mag, axis=-1, kind="stable")[..., :n_out]   # equal magnitudes: lower channel first
    vals = np.take_along_axis(XK, order, axis=-1)
    dense = XK.copy()
    np.put_along_axis(dense, order, np.uint16(0), axis=-1)
    return order, vals, dense


def quantize_kv_sparse(XK, XV, dtype, G, Gv, bits, symmetric=False, n_out=0) -> dict:
    """quantize_kv of the dense keys; "Ko" holds each token's outliers as words
    (channel << 16) | element bits, [BH, T, n_out], largest magnitude first."""
    if n_out == 0:
        q = quantize_kv(XK, XV, dtype, G, Gv, bits, symmetric)
        q["Ko"] = np.zeros(XK.shape[:2] + (0,), np.uint32)
        return q
    idx, vals, dense = key_outliers(XK, n_out, dtype)
    q = quantize_kv(dense, XV, dtype, G, Gv, bits, symmetric)
    q["Ko"] = (idx.astype(np.uint32) << 16) | vals.astype(np.uint32)
    return q


def dequantize(qc: dict, G: int, Gv: int, bits: int, symmetric: bool, dtype: int):
    """fp64 keys and values [BH, T, d] of a quantized block: x' = (q - z) s, plus the
    sparse key outliers at their channels."""
    z_sym = 1 << (bits - 1)
    Kz = np.full(qc["Ks"].shape, z_sym) if symmetric else qc["Kz"]
    Vz = np.full(qc["Vs"].shape, z_sym) if symmetric else qc["Vz"]
    K = (qc["Kq"].astype(np.float64) - np.repeat(Kz, G, axis=1)) * np.repeat(qc["Ks"].astype(np.float64), G, axis=1)
    V = (qc["Vq"].astype(np.float64) - np.repeat(Vz, Gv, axis=2)) * np.repeat(qc["Vs"].astype(np.float64), Gv, axis=2)
    Ko = qc.get("Ko")
    if Ko is not None and Ko.shape[-1]:
        ch = (Ko >> 16).astype(np.int64)
        x = widen_array((Ko & 0xFFFF).astype(np.uint16), dtype)
        np.put_along_axis(K, ch, np.take_along_axis(K, ch, axis=-1) + x, axis=-1)
    return K, V


def attend(K: np.ndarray, V: np.ndarray, Q: np.ndarray, dtype: int, B: int, Hq: int, Hkv: int) -> np.ndarray:
    """fp64 softmax(q k^T / sqrt(d)) v for queries Q bits [B, Hq, d] over K, V [B*Hkv, T, d]."""
    d = K.shape[-1]
    g = Hq // Hkv
    q = widen_array(Q, dtype).reshape(B, Hkv, g, d)
    K = K.reshape(B, Hkv, -1, d)
    V = V.reshape(B, Hkv, -1, d)
    s = np.einsum("bhgd,bhtd->bhgt", q, K) / np.sqrt(d)
    s -= s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return np.einsum("bhgt,bhtd->bhgd", p, V).reshape(B, Hq, d)


class SparseKeyCache(OracleCache):
    """OracleCache whose quantized keys keep n_out sparse outliers per token."""

    def __init__(self, B, Hq, Hkv, d, G, Gv, R, bits, symmetric=False, dtype=BF16, n_out=1):
        super().__init__(B, Hq, Hkv, d, G, Gv, R, bits, symmetric, dtype)
        self.n_out = n_out

    def _quantize_block(self, XK, XV):
        blk = quantize_kv_sparse(XK, XV, self.dtype, self.G, self.Gv, self.bits, self.symmetric, self.n_out)
        self.blocks.append(blk)
        self.Tq += XK.shape[1]
        self._cat = None

    def packed(self) -> dict:
        p = super().packed()
        qc = self.quantized()
        p["Ko"] = qc["Ko"] if "Ko" in qc else np.zeros((self.B * self.Hkv, 0, self.n_out), np.uint32)
        return p

    def decode(self, Q: np.ndarray, stats: bool = False):
        assert not stats
        BH = self.B * self.Hkv
        if self.Tq:
            Kd, Vd = dequantize(self.quantized(), self.G, self.Gv, self.bits, self.symmetric, self.dtype)
        else:
            Kd = Vd = np.zeros((BH, 0, self.d))
        K = np.concatenate([Kd, widen_array(self.Kr[:, :self.r], self.dtype)], axis=1)
        V = np.concatenate([Vd, widen_array(self.Vr[:, :self.r], self.dtype)], axis=1)
        return attend(K, V, Q, self.dtype, self.B, self.Hq, self.Hkv)
