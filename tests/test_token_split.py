"""Token-split decode on CPU: the shard plan, the oracle's merge of shard decodes
against the full-cache decode (the order-free concatenation of the LogQuant
summary, section 4), and the exchange between two gloo ranks."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_kv_cache_22_b200 import token_split
from bit_kv_cache_22_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("T,world,R", [(0, 2, 32), (5, 2, 32), (32, 2, 32), (300, 2, 32), (300, 3, 64),
                                       (4096, 8, 128), (100, 1, 32)])
def test_shard_bounds(T, world, R):
    b = token_split.shard_bounds(T, world, R)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == T
    for (lo, hi), (lo2, _) in zip(b, b[1:]):
        assert hi == lo2 and (hi - lo) % R == 0 and hi >= lo
    sizes = [hi - lo for lo, hi in b]
    assert max(sizes[:-1] or [0]) <= -(-T // world) + R      # balanced to within one residual


def _shard_caches(w, XK, XV, tK, tV, world):
    """Oracle caches of the shards (the last one takes every appended token)."""
    import kvq_testlib as tl
    caches = []
    for k, (lo, hi) in enumerate(token_split.shard_bounds(w.T, world, w.R)):
        c = tl.new_oracle(w)
        c.prefill(np.ascontiguousarray(XK[:, :, lo:hi]), np.ascontiguousarray(XV[:, :, lo:hi]))
        if k == world - 1:
            for s in range(w.steps):
                c.append(tK[s], tV[s])
        caches.append(c)
    return caches


@pytest.mark.parametrize("world", [2, 3])
def test_oracle_merge_of_shards_equals_full_decode(world):
    import kvq_testlib as tl
    import oracle
    w = wl.WORKLOADS["stream2"].replace(B=2, Hkv=2, Hq=8, T=3 * 128 + 40, steps=7)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    full = tl.new_oracle(w)
    full.prefill(XK, XV)
    for s in range(w.steps):
        full.append(tK[s], tV[s])
    want = full.decode(tQ[-1])
    parts = [c.decode(tQ[-1], stats=True) for c in _shard_caches(w, XK, XV, tK, tV, world) if c.Tq + c.r > 0]
    got = oracle.merge_partials([p[0] for p in parts], [p[1] for p in parts], [p[2] for p in parts])
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.WORKLOADS["tiny"].replace(T=200, steps=5)
        XK, XV = wl.prefill_bits(w)
        tK, tV, tQ = wl.decode_bits(w)
        mine = _shard_caches(w, XK, XV, tK, tV, world)[rank]
        o, m, l = mine.decode(tQ[-1], stats=True)
        # this rank's partial in the library's convention: base-2 logits, o unnormalised
        o2 = torch.from_numpy(o * l[..., None])
        m2 = torch.from_numpy(m * math.log2(math.e))
        l2 = torch.from_numpy(l)
        o_all, m_all, l_all = token_split.exchange_partials(o2, m2, l2)
        M = m_all.max(dim=0).values
        wgt = torch.exp2(m_all - M)
        merged = (o_all * wgt[..., None]).sum(0) / (l_all * wgt).sum(0)[..., None]
        out[rank] = merged.numpy()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_and_merge():
    import kvq_testlib as tl
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    w = wl.WORKLOADS["tiny"].replace(T=200, steps=5)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    full = tl.new_oracle(w)
    full.prefill(XK, XV)
    for s in range(w.steps):
        full.append(tK[s], tV[s])
    want = full.decode(tQ[-1])
    for r in range(world):               # every rank ends with the whole output
        np.testing.assert_allclose(out[r], want, rtol=1e-10, atol=1e-12)
