"""Benchmark: decode attention over a KIVI-style low-bit KV cache on B200.

One step = one full pass of the hot path over one batch: prefill-quantize the
prompt (keys per channel, values per token, residual tail), then every decode
step of the workload (append the new token -- flushing the residual when it
holds R tokens -- and split-K decode attention whose last split merges the partials).
The metric is KV tokens attended per second: each decode step attends to
B * (Tq + r) cached tokens.

Default workload: gqa8b, the largest single-GPU configuration (B32, 32 q / 8 kv
heads, d128, 8192-token prompt bf16, 2-bit asymmetric, G = Gv = 32, R = 128, 64
decode steps); a 1-GPU run adds long131k, llama7b, stream2 and stream4sym under
"workloads", each with its own roofline.  Multi-GPU runs are weak-scaled: every
rank serves its own batch of sequences (no data-path collective).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
       python bench.py --impl reference ...   (the CPU oracle, rank 0 only)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attn: KV tokens/s and achieved HBM GB/s vs B200 peak"
UNIT = "KV tokens/s"
FALLBACK_HBM_GBS = 6650.0


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default="gqa8b")
    p.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="measure the headline workload only (by default a 1-GPU run adds the others)")
    p.add_argument("--ncu-case", action="store_true",
                   help="run one prefill and up to 64 decode steps of the workload, then exit (for ncu)")
    p.add_argument("--paged", default=None, metavar="RAGGED_WORKLOAD",
                   help="measure the paged, ragged cache on this ragged batch (e.g. ragged_gqa) instead")
    p.add_argument("--window", type=int, default=0,
                   help="measure LogQuant retention with this window W on the workload instead")
    p.add_argument("--key-outliers", type=int, default=0,
                   help="dense-and-sparse keys: keep this many outliers per token (1 or 2)")
    p.add_argument("--decode-kernel", default="auto", choices=list(DECODE_KERNELS),
                   help="the decode kernel (kvq_set_decode_kernel): the library's choice or one forced")
    return p.parse_args()


# --decode-kernel: the kvq_set_decode_kernel value and the kernel it launches
DECODE_KERNELS = {"auto": (0, None), "cuda-cores": (1, "decode_split_kernel"),
                  "int8-mma": (2, "decode_tc_kernel"), "bf16-mma": (3, "decode_mma_kernel")}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def algorithmic_bytes(w, Tq: int, r: int) -> int:
    """Bytes one decode attention must move: packed codes, scales/zeros, residual
    rows, the query and the fp32 output."""
    BH = w.B * w.Hkv
    meta = 4 if w.symmetric else 6
    # codes of K and V, key meta amortised over its G tokens, value meta per token
    per_tok = 2 * w.d * w.bits / 8 + w.d * meta / w.G + (w.d // w.Gv) * meta
    return int(BH * (Tq * per_tok + r * 2 * w.d * 2) + w.B * w.Hq * w.d * (2 + 4))


def episode_contexts(w):
    """(Tq, r) seen by each decode step of an episode."""
    out = []
    Tq, r = (w.T // w.R) * w.R, w.T % w.R
    for _ in range(w.steps):
        r += 1
        if r == w.R:
            Tq, r = Tq + w.R, 0
        out.append((Tq, r))
    return out


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_kernel_name(w, paged: bool = False, key_outliers: int = 0, forced: str = "auto") -> str:
    """The decode kernel the library launches for this geometry."""
    if DECODE_KERNELS[forced][1]:
        return DECODE_KERNELS[forced][1]
    if w.Hq // w.Hkv not in (1, 2, 4) or w.G < 32:
        return "decode_split_kernel"
    return "decode_tc_kernel" if paged or key_outliers else "decode_mma_kernel"


# the sources a decode kernel's code comes from (a profile names their hash)
KERNEL_SOURCES = {
    "decode_mma_kernel": ("decode_mma.cuh", "decode_kernels.cuh"),
    "decode_tc_kernel": ("decode_kernels.cuh",),
    "decode_split_kernel": ("decode_kernels.cuh",),
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "bit_kv_cache_22_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(w, kernel=None):
    """Per-launch DRAM bytes of the decode kernel from the committed ncu summary,
    if it was taken on the current kernel source (else None)."""
    kernel = kernel or decode_kernel_name(w)
    path = os.path.join(ROOT, "profiles", f"{kernel}_{w.name}.md")
    try:
        text = open(path).read()
        m_sha = re.search(r"kernel source sha256\[:16\]:\s*([0-9a-f]{16})", text)
        m_b = re.search(r"dram bytes per launch:\s*([0-9]+)", text)
        if m_sha and m_b and m_sha.group(1) == kernel_source_hash(kernel):
            return int(m_b.group(1))
    except OSError:
        pass
    return None


def shard_workload(base, rank: int):
    """Weak scaling: every rank serves its own batch of sequences (seed offset by rank)."""
    return base if rank == 0 else base.replace(seed=base.seed + 1000 * rank)


def max_over_ranks(values, world: int, device=None):
    """Element-wise maximum of per-rank values (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_throughput(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the library arm
# ---------------------------------------------------------------------------

L2_BYTES = 126 * 1024 * 1024      # B200 L2 (126 MB): per-call inputs below it are timed L2-scrubbed
EXTRA_WORKLOADS = ("long131k", "llama7b", "stream2", "stream4sym")


class L2Scrub:
    """A read of 2 x L2 bytes: evicts whatever the previous call left in L2 and leaves
    clean lines behind (nothing to write back during the next timed call)."""

    def __init__(self, dev):
        import torch
        self.buf = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        torch.sum(self.buf, dim=0, out=self.out)


def _replay_ms(graph, k, stream):
    """Device time of k back-to-back replays of a CUDA graph (two events on the stream)."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(k):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def measure_workload(w, args, dev, local, world, headline: bool):
    """One workload on this rank: whole-episode throughput (value), per-decode-call time and
    the roofline, and (headline only) the end-to-end figure through the public API.

    The episode (prefill + every decode step) is captured as one CUDA graph and replayed
    K times between two events: `value` and `ms_per_step`.  The decode calls alone -- every
    step's append_decode (at a flush: append, then decode) after the prompt's prefill -- are
    a second graph, replayed K times back to back; replaying it is idempotent (every step
    rewrites the residual row and the flushed tokens it wrote before).  A third graph holds
    only the flush steps' appends; per call = (decode graph - flush graph) / steps, so
    avg_launch_us x steps <= ms_per_step.  When one call's cache fits in L2, every decode
    step in the decode graph is preceded by a read of a 2 x L2 buffer, and the time of a
    graph of those reads alone is subtracted too: `cold` timing."""
    import torch
    import torch.distributed as dist

    from bit_kv_cache_22_b200 import kvq
    from bit_kv_cache_22_b200 import workloads as wl

    dt = torch.float16 if w.dtype == wl.FP16 else torch.bfloat16

    def to_t(bits, pin=False):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt)
        return t.pin_memory() if pin else t

    XK_h, XV_h = wl.prefill_bits(w)
    tK_h, tV_h, tQ_h = wl.decode_bits(w)
    XK, XV = to_t(XK_h).to(dev), to_t(XV_h).to(dev)
    tK, tV, tQ = to_t(tK_h).to(dev), to_t(tV_h).to(dev), to_t(tQ_h).to(dev)
    cache = kvq.KVQCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, dt,
                         w.capacity, dev, key_outliers=args.key_outliers)
    cache.set_decode_kernel(DECODE_KERNELS[args.decode_kernel][0])
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    ctx = episode_contexts(w)
    call_bytes = [algorithmic_bytes(w, tq, r) + w.B * w.Hkv * tq * 4 * args.key_outliers for tq, r in ctx]
    tokens_per_episode = sum(w.B * (tq + r) for tq, r in ctx)
    cold = max(call_bytes) < L2_BYTES
    scrub = L2Scrub(dev) if cold else None

    def episode():
        cache.reset()
        cache.prefill_quantize(XK, XV)
        for s in range(w.steps):
            cache.append_decode(tK[s], tV[s], tQ[s], out=out)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        episode()
    torch.cuda.synchronize()
    pool = torch.cuda.graph_pool_handle()
    launches0 = kvq.kernel_launches()
    cache.reset()
    g_ep = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ep, pool=pool):
        episode()
    launches_per_episode = kvq.kernel_launches() - launches0
    # the decode calls after an eager prefill, and (separately) the flush steps' appends
    cache.reset()
    cache.prefill_quantize(XK, XV)
    torch.cuda.synchronize()
    flush_steps = []
    g_dec = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_dec, pool=pool):
        for s in range(w.steps):
            if cache.state()[1] + 1 == w.R:
                flush_steps.append(s)
                cache.append(tK[s], tV[s])
                if scrub:
                    scrub()
                cache.decode_attention(tQ[s], out=out)
            else:
                if scrub:
                    scrub()
                cache.append_decode(tK[s], tV[s], tQ[s], out=out)
    # what the decode graph holds besides the decode calls: each flush step's append (its own
    # graph, captured at that step's state: the steps in between run eagerly) and the scrubs
    side = []
    if flush_steps:
        cache.reset()
        cache.prefill_quantize(XK, XV)
        for s in range(w.steps):
            if s in flush_steps:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, pool=pool):
                    cache.append(tK[s], tV[s])
                g.replay()
                side.append(g)
            else:
                cache.append(tK[s], tV[s])
    if scrub:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, pool=pool):
            for s in range(w.steps):
                scrub()
        side.append(g)
    torch.cuda.synchronize()

    def replay_side():
        for g in side:
            g.replay()

    with ClockSampler(local) as clk:
        g_ep.replay()
        g_dec.replay()
        replay_side()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        # timed region: K episodes, each one whole-episode graph replay
        ms = _replay_ms(g_ep, args.steps, stream)
        barrier()
        dec_ms = _replay_ms(g_dec, args.steps, stream)
        side_ms = 0.0
        if side:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                replay_side()
            e1.record(stream)
            torch.cuda.synchronize()
            side_ms = e0.elapsed_time(e1)
        barrier()
    launches = launches_per_episode * args.steps
    decode_ms = max(dec_ms - side_ms, 1e-6)
    ms, decode_ms = max_over_ranks([ms, decode_ms], world, dev)
    del g_dec, side

    e2e = None
    if headline and not args.no_e2e:
        XKp, XVp = to_t(XK_h, True), to_t(XV_h, True)
        tKp, tVp, tQp = to_t(tK_h, True), to_t(tV_h, True), to_t(tQ_h, True)
        outs = torch.empty((w.steps, w.B, w.Hq, w.d), dtype=torch.float32).pin_memory()

        def e2e_episode():
            cache.reset()
            cache.prefill_quantize(XKp, XVp)           # host -> device inside the call path
            for s in range(w.steps):
                cache.append_decode(tKp[s], tVp[s], tQp[s], out=outs[s])   # device -> host of t_O
        for _ in range(max(1, args.warmup)):
            e2e_episode()
        torch.cuda.synchronize()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            e2e_episode()
        g2.replay()
        torch.cuda.synchronize()
        barrier()
        e2e_ms, = max_over_ranks([_replay_ms(g2, args.steps, stream)], world, dev)
        barrier()
        h2d = XKp.numel() * 2 * 2 + w.steps * (2 * w.B * w.Hkv * w.d + w.B * w.Hq * w.d) * 2
        d2h = w.steps * w.B * w.Hq * w.d * 4
        e2e = {"value": job_throughput(tokens_per_episode * args.steps, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / args.steps}
        del g2

    peak, peak_kind = peaks()
    kname = decode_kernel_name(w, key_outliers=args.key_outliers, forced=args.decode_kernel)
    per_call_ms = decode_ms / (args.steps * w.steps)
    bytes_per_call = sum(call_bytes) / w.steps
    achieved = bytes_per_call / (per_call_ms / 1e3) / 1e9
    res = {
        "workload": w.name,
        "value": job_throughput(tokens_per_episode * args.steps, world, ms),
        "ms_per_step": ms / args.steps,
        "decode_steps_per_s": w.steps * args.steps / (ms / 1e3),
        "kv_tokens_per_s_decode_only": job_throughput(tokens_per_episode * args.steps, world, decode_ms),
        "splits": cache.splits(),
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "e2e": e2e,
        "roofline": {
            "kernel": f"append + decode_attention ({kname}: one launch without a flush, "
                      "splits merged in-kernel), per call",
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
            if peak_kind == "measured" else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_launch": bytes_per_call,
            "avg_launch_us": per_call_ms * 1e3,
            "l2": "cold: a read of 2 x L2 before every timed call (its time subtracted)" if cold else
                  "inputs larger than L2 (calls back to back)",
            "timing_ms": {"decode_graph": dec_ms, "side_graph": side_ms, "replays": args.steps},
            "traffic": ncu_traffic(w, kname),
        },
        "config": {
            "workload": w.name, "batch_per_gpu": w.B, "global_batch": w.B * world,
            "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d, "prompt_tokens": w.T,
            "decode_steps": w.steps, "bits": w.bits, "group_k": w.G, "group_v": w.Gv,
            "residual": w.R, "symmetric": w.symmetric, "key_outliers_per_token": args.key_outliers,
            "elem": "fp16" if w.dtype == wl.FP16 else "bf16",
            "decode_kernel": kname,
        },
    }
    del cache, XK, XV, tK, tV, tQ, g_ep, scrub
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_kvq(args):
    import torch
    import torch.distributed as dist

    from bit_kv_cache_22_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    w = shard_workload(wl.WORKLOADS[args.workload], rank)

    if args.ncu_case:
        from bit_kv_cache_22_b200 import kvq
        dt = torch.float16 if w.dtype == wl.FP16 else torch.bfloat16

        def to_t(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).to(dev)
        XK, XV = (to_t(x) for x in wl.prefill_bits(w))
        tK, tV, tQ = (to_t(x) for x in wl.decode_bits(w))
        cache = kvq.KVQCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, dt,
                             w.capacity, dev, key_outliers=args.key_outliers)
        cache.set_decode_kernel(DECODE_KERNELS[args.decode_kernel][0])
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
        cache.prefill_quantize(XK, XV)
        for s in range(min(w.steps, 64)):      # ends mid-episode (r = 64 residual rows at most)
            cache.append_decode(tK[s], tV[s], tQ[s], out=out)
        torch.cuda.synchronize()
        print(json.dumps({"ncu_case": args.workload, "state": cache.state()}))
        return

    head = measure_workload(w, args, dev, local, world, headline=True)
    extras = {}
    if world == 1 and not args.no_extra:
        for name in EXTRA_WORKLOADS:
            if name != w.name:
                extras[name] = measure_workload(wl.WORKLOADS[name], args, dev, local, world, headline=False)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, budget_s=20.0)

    config = dict(head["config"])
    config.update({
        "parallelism": f"dp{world} (independent sequences per GPU)",
        "splits": head["splits"],
        "l2": head["roofline"]["l2"],
        "timing": "value: K whole-episode CUDA-graph replays (prefill + every decode step) between two "
                  "events; roofline: events inside one graph of the episode's decode calls, K replays",
    })
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"u{w.bits} codes, f32 accumulate",
        "data": "synthetic (seeded; distributions of the workload definition)",
        "config": config,
        "decode_steps_per_s": head["decode_steps_per_s"],
        "kv_tokens_per_s_decode_only": head["kv_tokens_per_s_decode_only"],
        "roofline": head["roofline"],
        "cpu_baseline": cpu,
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "workloads": {name: {k: r[k] for k in ("value", "ms_per_step", "decode_steps_per_s", "roofline",
                                                "splits", "gpu_launches", "clocks", "config")}
                      for name, r in extras.items()},
    }
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# decode-only measurements: LogQuant retention and the paged, ragged cache
# ---------------------------------------------------------------------------

def _rank_setup(args):
    """(world, rank, local rank, device) of this process; NCCL process group for N > 1."""
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))
    return world, rank, local, dev


def _time_decode_steps(args, cache, steps, tK, tV, tQ, out, local, count):
    """Per decode step: an eager append, then the step's decode_attention captured as a CUDA
    graph, warmed up and replayed `--steps` times between two events on the replay stream.
    count() gives (KV tokens, algorithmic bytes) of one decode call at the current state.
    Returns (decode ms, KV tokens, bytes, kernel launches, clock sampler)."""
    import torch

    from bit_kv_cache_22_b200 import kvq

    stream = torch.cuda.current_stream()
    pool = torch.cuda.graph_pool_handle()
    total_ms, total_tokens, total_bytes, launches = 0.0, 0, 0, 0
    with ClockSampler(local) as clk:
        for s in range(steps):
            cache.append(tK[s], tV[s])
            torch.cuda.synchronize()
            l0 = kvq.kernel_launches()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, pool=pool):
                cache.decode_attention(tQ[s], out=out)
            per_call = kvq.kernel_launches() - l0
            for _ in range(max(1, args.warmup)):
                g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            total_ms += e0.elapsed_time(e1)
            launches += per_call * args.steps
            tokens, nbytes = count()
            total_tokens += tokens * args.steps
            total_bytes += nbytes * args.steps
            del g
    return total_ms, total_tokens, total_bytes, launches, clk


def _decode_only_line(args, w, world, ms, total_ms, total_tokens, total_bytes, launches, clk, config,
                      kernel):
    """The JSON line of a decode-only measurement (rank 0)."""
    from bit_kv_cache_22_b200 import workloads as wl

    calls = w.steps * args.steps
    peak, peak_kind = peaks()
    achieved = total_bytes / (total_ms / 1e3) / 1e9
    config = dict(config)
    config.update({
        "elem": "fp16" if w.dtype == wl.FP16 else "bf16", "parallelism": f"dp{world}",
        "l2": f"inputs larger than L2: packed cache {total_bytes / calls / 1e6:.0f} MB per decode call",
        "timing": "per decode step: its decode_attention graph replayed --steps times between "
                  "two events (value and roofline: decode time only; appends run eagerly between)",
    })
    return {
        "metric": METRIC, "value": job_throughput(total_tokens, world, ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / calls,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"u{w.bits} codes, f32 accumulate",
        "data": "synthetic (seeded; distributions of the workload definition)",
        "config": config,
        "roofline": {
            "kernel": kernel, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak,
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_launch": total_bytes / calls, "avg_launch_us": total_ms / calls * 1e3,
            "traffic": None,
        },
        "cpu_baseline": None,
        "e2e": None,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }


def _finish(world, rank, line):
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_logquant(args):
    """Decode attention with LogQuant retention (window W) on the workload's batch: the
    prompt's prefill (eager: it uploads row lists), then the decode steps timed by
    _time_decode_steps.  value = KV tokens attended per second of decode time; the roofline
    counts the quantized tokens' bytes and the full-precision store's rows."""
    import torch

    from bit_kv_cache_22_b200 import kvq
    from bit_kv_cache_22_b200 import workloads as wl

    world, rank, local, dev = _rank_setup(args)
    w = shard_workload(wl.WORKLOADS[args.workload], rank)
    W = args.window
    dt = torch.float16 if w.dtype == wl.FP16 else torch.bfloat16

    def to_t(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).to(dev)

    cap = -(-(w.T + w.steps) // W) * W
    cache = kvq.KVQCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, dt, cap, dev,
                         window=W, key_outliers=args.key_outliers)
    cache.set_decode_kernel(DECODE_KERNELS[args.decode_kernel][0])
    kname = decode_kernel_name(w, key_outliers=args.key_outliers, forced=args.decode_kernel)
    XK, XV = wl.prefill_bits(w)
    cache.prefill_quantize(to_t(XK), to_t(XV))
    del XK, XV
    tK, tV, tQ = (to_t(x) for x in wl.decode_bits(w))
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)

    def count():
        tq, r = cache.state()
        return w.B * (tq + r), algorithmic_bytes(w, tq, r) + w.B * w.Hkv * tq * 4 * args.key_outliers

    total_ms, tokens, nbytes, launches, clk = _time_decode_steps(args, cache, w.steps, tK, tV, tQ, out, local,
                                                                 count)
    ms, = max_over_ranks([total_ms], world, dev)
    tq, r = cache.state()
    config = {"workload": f"{w.name} (LogQuant retention, W={W})", "batch_per_gpu": w.B, "q_heads": w.Hq,
              "kv_heads": w.Hkv, "head_dim": w.d, "prompt_tokens": w.T, "decode_steps": w.steps,
              "bits": w.bits, "group_k": w.G, "group_v": w.Gv, "window": W,
              "key_outliers_per_token": args.key_outliers, "full_precision_rows_at_end": r,
              "splits": cache.splits()}
    line = _decode_only_line(args, w, world, ms, total_ms, tokens, nbytes, launches, clk, config,
                             f"decode_attention ({kname}) over a LogQuant cache, per call")
    _finish(world, rank, line)


def run_paged(args):
    """Decode attention of a ragged batch held in a paged cache.  After the prompts'
    prefill, every decode step appends one token per slot (eagerly: the page table is
    written from the host when a flush opens a page) and is timed by _time_decode_steps.
    value = KV tokens attended per second of decode time over all steps; the roofline uses
    the algorithmic bytes of every slot at its own length."""
    import torch

    from bit_kv_cache_22_b200 import kvq
    from bit_kv_cache_22_b200 import workloads as wl

    world, rank, local, dev = _rank_setup(args)
    spec = wl.RAGGED[args.paged]
    w = shard_workload(spec["base"], rank)
    lens = wl.ragged_lengths(w, spec["lo"], spec["hi"])
    P = spec["page_tokens"]
    dt = torch.float16 if w.dtype == wl.FP16 else torch.bfloat16

    def to_t(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).to(dev)

    cap = -(-(max(lens) + w.steps) // P) * P
    cache = kvq.PagedKVQCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, dt, cap, P,
                              None, dev)
    np.random.default_rng(w.seed).shuffle(cache.free_pages)     # a scrambled pool
    for b, T in enumerate(lens):
        XK, XV = wl.prefill_bits(w, bs=[b], T=T)
        cache.prefill(b, to_t(XK[0]), to_t(XV[0]))
    tK, tV, tQ = (to_t(x) for x in wl.decode_bits(w))
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    w1 = w.replace(B=1)

    def count():
        n = [cache.lens[b] for b in range(w.B)]
        return sum(n), sum(algorithmic_bytes(w1, x // w.R * w.R, x % w.R) for x in n)

    total_ms, tokens, nbytes, launches, clk = _time_decode_steps(args, cache, w.steps, tK, tV, tQ, out, local,
                                                                 count)
    ms, = max_over_ranks([total_ms], world, dev)
    config = {"workload": f"{args.paged} (paged, ragged)", "slots_per_gpu": w.B, "q_heads": w.Hq,
              "kv_heads": w.Hkv, "head_dim": w.d,
              "prompt_tokens": f"{min(lens)}..{max(lens)} (mean {sum(lens) / len(lens):.0f})",
              "page_tokens": P, "decode_steps": w.steps, "bits": w.bits, "group_k": w.G, "group_v": w.Gv,
              "residual": w.R, "splits": cache.splits()}
    line = _decode_only_line(args, w, world, ms, total_ms, tokens, nbytes, launches, clk, config,
                             f"paged decode_attention ({decode_kernel_name(w, paged=True)}, paged instance), per call")
    _finish(world, rank, line)


# ---------------------------------------------------------------------------
# the CPU oracle (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's processor string."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_sample(w, budget_s, XK, XV, tK, tV, tQ):
    """One timed oracle run: prefill of one sequence, then decode steps until budget_s."""
    import oracle
    t0 = time.perf_counter()
    c = oracle.OracleCache(1, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, w.dtype)
    c.prefill(XK, XV)
    tokens, done = 0, 0
    for s in range(w.steps):
        c.append(tK[s], tV[s])
        c.decode(tQ[s])
        tokens += c.Tq + c.r
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return tokens, done, time.perf_counter() - t0


def cpu_baseline(w, budget_s=20.0, one_core_s=8.0):
    """Time the oracle (as it stands) on a bounded sample of the workload: one
    sequence (all of its kv heads), its prompt prefill and the first decode
    steps, stopping after ~budget_s seconds, on all the threads the oracle uses;
    then the same sample on one thread for ~one_core_s seconds.  KV tokens/s."""
    import oracle
    from bit_kv_cache_22_b200 import workloads as wl
    XK, XV = wl.prefill_bits(w, bs=[0])
    tK, tV, tQ = wl.decode_bits(w, bs=[0])
    threads = oracle.num_threads()
    tokens, done, el = _oracle_sample(w, budget_s, XK, XV, tK, tV, tQ)
    res = {"value": tokens / el, "unit": UNIT, "cores": threads, "kind": "oracle",
           "cpu_model": cpu_model(), "host_cores": len(os.sched_getaffinity(0)),
           "sample": f"1 of {w.B} sequences (all {w.Hkv} kv heads): prefill of {w.T} tokens + "
                     f"{done} of {w.steps} decode steps, {el:.1f} s, fp64 C oracle with OpenMP "
                     f"on {threads} threads"}
    if one_core_s > 0:
        old = oracle.set_num_threads(1)
        try:
            t1, d1, e1 = _oracle_sample(w, one_core_s, XK, XV, tK, tV, tQ)
        finally:
            oracle.set_num_threads(old)
        res["one_core"] = {"value": t1 / e1, "unit": UNIT, "cores": 1,
                           "sample": f"the same sample on 1 thread: prefill + {d1} decode steps, {e1:.1f} s"}
    return res


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from bit_kv_cache_22_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(w, budget_s=budget, one_core_s=0)
    vals = [cpu_baseline(w, budget_s=budget, one_core_s=0) for _ in range(args.steps)]
    v = statistics.mean(x["value"] for x in vals)
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "impl": "reference", "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": w.name, "global_batch": w.B, "note": "CPU oracle, rank 0"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": vals[0]["cores"],
                             "cpu_model": vals[0]["cpu_model"], "host_cores": vals[0]["host_cores"],
                             "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    elif args.paged:
        run_paged(args)
    elif args.window:
        run_logquant(args)
    else:
        run_kvq(args)


if __name__ == "__main__":
    main()
