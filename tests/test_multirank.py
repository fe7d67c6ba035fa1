"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

Each rank serves its own batch (weak scaling, no data-path collective); the
job time is the maximum over ranks and the throughput counts every rank's
units.  Runs as two spawned processes with the gloo backend on 127.0.0.1.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from bit_kv_cache_22_b200 import workloads as wl
        w = bench.shard_workload(wl.WORKLOADS["llama7b"], rank)
        k, _ = wl.prefill_slice(w, 0, 0, T=4)
        times = [10.0 + 5.0 * rank, 3.0 - rank]          # rank 1 is slower in the first value
        mx = bench.max_over_ranks(times, world)
        out[rank] = (w.seed, float(k[0, 0]), mx,
                     bench.job_throughput(1000.0, world, mx[0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    (s0, k0, mx0, v0), (s1, k1, mx1, v1) = out[0], out[1]
    assert s0 != s1 and k0 != k1                  # independent sequences per rank
    assert mx0 == mx1 == [15.0, 3.0]              # every rank sees the slowest rank's time
    assert v0 == v1 == pytest.approx(1000.0 * 2 / 0.015)
