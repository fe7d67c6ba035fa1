"""The decode split planner on the host (kvq_plan_decode, the function every decode
call uses): its coverage and size invariants over random geometries and ragged
lengths, and the plans of the measured workloads."""
import numpy as np
import pytest

from bit_kv_cache_22_b200 import kvq


def _cfg(B, Hq, Hkv, d, G, Gv, R, bits, cap):
    return kvq.make_config(B, Hq, Hkv, d, G, Gv, R, bits, False, kvq.KVQ_BF16, cap)


def test_measured_workloads_plans():
    # contiguous caches with 1, 2 or 4 query heads per kv head: the bf16-MMA kernel, items of
    # two tiles, residual rows in splits of their own
    llama = _cfg(8, 32, 32, 128, 128, 128, 128, 4, 4352)
    nq, per, S = kvq.plan_decode(llama, [4096 + 21] * 8, 148, 3)
    assert per % 2 == 0 and nq * per >= 256 > (nq - 1) * per and S > nq
    gqa = _cfg(32, 32, 8, 128, 32, 32, 128, 2, 8320)
    nq, per, S = kvq.plan_decode(gqa, [8192 + 21] * 32, 148, 3)
    assert per % 2 == 0 and nq * per >= 512 > (nq - 1) * per and S > nq


@pytest.mark.parametrize("seed", range(40))
def test_plan_invariants(seed):
    rng = np.random.default_rng(seed)
    g = int(rng.choice([1, 2, 4, 8]))
    Hkv = int(rng.choice([1, 2, 8]))
    G = int(rng.choice([16, 32, 64, 128]))
    R = G * int(rng.choice([1, 2, 4]))
    d = int(rng.choice([64, 128]))
    B = int(rng.integers(1, 40))
    cap = R * int(rng.integers(1, 400))
    ragged = bool(rng.integers(0, 2))
    if ragged:
        lens = [int(x) for x in rng.integers(-1, cap + R - 1, B)]
    else:
        lens = [int(rng.integers(0, cap + R - 1))] * B
    cfg = _cfg(B, g * Hkv, Hkv, d, G, min(G, d), R, 2, cap)
    nq, per, S = kvq.plan_decode(cfg, lens, int(rng.choice([1, 20, 148])), int(rng.integers(1, 5)))
    tiles = [max(x, 0) // R * R // 16 for x in lens]
    rres = max(max(x, 0) % R for x in lens)
    tc = g in (1, 2, 4) and G >= 32
    assert S >= 1 and S - nq <= 16 and nq <= 128
    assert S <= min(cap // 16, 128) + 16                   # the workspace's bound
    if max(tiles) > 0:
        assert nq * per >= max(tiles) > (nq - 1) * per     # every tile covered, no empty last split
        if tc:
            assert per % 2 == 0                            # items of two tiles
    if rres > 0:
        assert S - nq >= 1
    else:
        assert S == nq


def test_plan_rejects_lengths_beyond_capacity():
    cfg = _cfg(2, 4, 2, 128, 32, 32, 64, 2, 256)
    with pytest.raises(kvq.KVQError):
        kvq.plan_decode(cfg, [100, 1000])
