"""Shared helpers of the GPU parity tests: run a workload through the C ABI and
through the oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

ATOL, RTOL = 2e-3, 1e-2     # output tolerance: |gpu - ref| <= ATOL + RTOL * |ref|


def torch_dtype(w: wl.Workload):
    return torch.float16 if w.dtype == wl.FP16 else torch.bfloat16


def to_dev(bits: np.ndarray, w: wl.Workload, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch_dtype(w)).to(device)


def new_cache(w: wl.Workload, capacity: int | None = None) -> kvq.KVQCache:
    return kvq.KVQCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric,
                        torch_dtype(w), capacity or w.capacity, "cuda")


def new_oracle(w: wl.Workload, B=None, Hq=None, Hkv=None):
    import oracle
    return oracle.OracleCache(B or w.B, Hq or w.Hq, Hkv or w.Hkv, w.d, w.G, w.Gv, w.R, w.bits,
                              w.symmetric, w.dtype)


def gpu_packed(cache: kvq.KVQCache, Tq: int, bh=None) -> dict:
    """Quantized part of the GPU cache in the oracle's array shapes (numpy)."""
    c = cache.cfg
    words = Tq * c.head_dim * c.bits // 32
    sel = slice(None) if bh is None else [bh]
    out = dict(
        Kc=cache.k_codes[sel, :words].cpu().numpy().view(np.uint32),
        Vc=cache.v_codes[sel, :words].cpu().numpy().view(np.uint32),
        Ks=cache.k_scales[sel, :Tq // c.group_k].cpu().numpy(),
        Vs=cache.v_scales[sel, :Tq].cpu().numpy())
    if cache.k_zeros is not None:
        out["Kz"] = cache.k_zeros[sel, :Tq // c.group_k].cpu().numpy()
        out["Vz"] = cache.v_zeros[sel, :Tq].cpu().numpy()
    return out


def assert_codes_equal(gpu: dict, ref: dict, symmetric: bool):
    keys = ("Kc", "Vc", "Ks", "Vs") + (() if symmetric else ("Kz", "Vz"))
    for k in keys:
        g, r = gpu[k], ref[k]
        assert g.shape == r.shape, (k, g.shape, r.shape)
        if g.dtype == np.float32:
            g, r = g.view(np.uint32), r.view(np.uint32)
        bad = np.argwhere(g != r)
        assert bad.size == 0, f"{k}: {len(bad)} mismatches, first at {bad[:3].tolist()}"


def assert_close(gpu: np.ndarray, ref: np.ndarray, what=""):
    err = np.abs(gpu.astype(np.float64) - ref)
    lim = ATOL + RTOL * np.abs(ref)
    bad = err > lim
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance, "
                           f"max err {err.max():.3e}, worst ratio {(err / lim).max():.2f}")
    return float(err.max())
