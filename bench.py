"""Benchmark: decode attention over a KIVI-style low-bit KV cache on B200.

One step = one full pass of the hot path over one batch: prefill-quantize the
prompt (keys per channel, values per token, residual tail), then every decode
step of the workload (append the new token -- flushing the residual when it
holds R tokens -- and split-K decode attention whose last split merges the partials).
The metric is KV tokens attended per second: each decode step attends to
B * (Tq + r) cached tokens.

Default workload: llama7b (B8, 32 MHA heads, d128, 4096-token prompt bf16,
4-bit asymmetric, G = Gv = R = 128, 128 decode steps).  Multi-GPU runs are
weak-scaled: every rank serves its own batch of 8 sequences (no data-path
collective).

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
    p.add_argument("--workload", default="llama7b")
    p.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--ncu-case", action="store_true",
                   help="run one prefill and up to 64 decode steps of the workload, then exit (for ncu)")
    p.add_argument("--paged", default=None, metavar="RAGGED_WORKLOAD",
                   help="measure the paged, ragged cache on this ragged batch (e.g. ragged_gqa) instead")
    p.add_argument("--window", type=int, default=0,
                   help="measure LogQuant retention with this window W on the workload instead")
    p.add_argument("--key-outliers", type=int, default=0,
                   help="dense-and-sparse keys: keep this many outliers per token (1 or 2)")
    return p.parse_args()


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


def decode_kernel_name(w) -> str:
    """The decode kernel the library launches for this geometry."""
    return "decode_tc_kernel" if w.Hq // w.Hkv in (1, 2, 4) and w.G >= 32 else "decode_split_kernel"


def ncu_traffic(w):
    """Per-launch DRAM bytes of the decode kernel from the committed ncu summary,
    if it was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{decode_kernel_name(w)}_{w.name}.md")
    src = os.path.join(ROOT, "bit_kv_cache_22_b200", "csrc", "decode_kernels.cuh")
    try:
        text = open(path).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        m_sha = re.search(r"decode_kernels\.cuh sha256\[:16\]:\s*([0-9a-f]{16})", text)
        m_b = re.search(r"dram bytes per launch:\s*([0-9]+)", text)
        if m_sha and m_b and m_sha.group(1) == sha:
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

def run_kvq(args):
    import torch
    import torch.distributed as dist

    from bit_kv_cache_22_b200 import kvq
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
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    if args.ncu_case:
        cache.prefill_quantize(XK, XV)
        for s in range(min(w.steps, 64)):      # ends with r = 64 residual rows, mid-episode
            cache.append_decode(tK[s], tV[s], tQ[s], out=out)
        torch.cuda.synchronize()
        print(json.dumps({"ncu_case": args.workload, "state": cache.state()}))
        return

    ctx = episode_contexts(w)
    tokens_per_episode = sum(w.B * (tq + r) for tq, r in ctx)
    bytes_per_episode = sum(algorithmic_bytes(w, tq, r) for tq, r in ctx)
    bytes_per_episode += sum(w.B * w.Hkv * tq * 4 * args.key_outliers for tq, r in ctx)   # outlier words

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
    # The episode is captured once as a sequence of CUDA graphs -- the prompt
    # prefill, then per decode step one graph for append (+ flush) and one for
    # decode_attention -- and replayed in that order: the host-side cost of
    # ~640 small launches per episode would otherwise starve the GPU.  Timing
    # events sit between the graph launches, on the capture/replay stream, so
    # every decode_attention call of the timed region is timed individually.
    launches0 = kvq.kernel_launches()
    pool = torch.cuda.graph_pool_handle()
    cache.reset()
    g_pre = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_pre, pool=pool):
        cache.prefill_quantize(XK, XV)
    # a step whose append flushes the residual gets its own append graph (the quantize is
    # not part of the timed decode); every other step is one append_decode graph
    g_app, g_dec = [], []
    for s_ in range(w.steps):
        flush = cache.state()[1] + 1 == w.R
        ga, gd = (torch.cuda.CUDAGraph() if flush else None), torch.cuda.CUDAGraph()
        if flush:
            with torch.cuda.graph(ga, pool=pool):
                cache.append(tK[s_], tV[s_])
            with torch.cuda.graph(gd, pool=pool):
                cache.decode_attention(tQ[s_], out=out)
        else:
            with torch.cuda.graph(gd, pool=pool):
                cache.append_decode(tK[s_], tV[s_], tQ[s_], out=out)
        g_app.append(ga)
        g_dec.append(gd)
    launches_per_episode = kvq.kernel_launches() - launches0
    # the whole episode as one graph: what `value` times
    cache.reset()
    g_ep = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ep, pool=pool):
        episode()
    torch.cuda.synchronize()

    def replay_episode(ev):
        g_pre.replay()
        for s_ in range(w.steps):
            if g_app[s_] is not None:
                g_app[s_].replay()
            ev[s_][0].record(stream)
            g_dec[s_].replay()
            ev[s_][1].record(stream)

    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(w.steps)] for _ in range(args.steps + 1)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        g_ep.replay()                    # graph warm-up (also gives the sampler time to start)
        replay_episode(evs[-1])
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        # timed region: K episodes, each one whole-episode graph replay
        start.record(stream)
        for k in range(args.steps):
            g_ep.replay()
        stop.record(stream)
        torch.cuda.synchronize()
        barrier()
        # the same K episodes replayed step by step, with events around every
        # decode_attention call: the per-call duration the roofline uses
        for k in range(args.steps):
            replay_episode(evs[k])
        torch.cuda.synchronize()
        barrier()
    launches = launches_per_episode * args.steps
    ms = start.elapsed_time(stop)
    decode_ms = sum(a.elapsed_time(b) for ev in evs[:args.steps] for a, b in ev)
    ms, decode_ms = max_over_ranks([ms, decode_ms], world, dev)

    # ---- end to end through the public API with pinned host buffers ----
    e2e = None
    if not args.no_e2e:
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
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            g2.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms, = max_over_ranks([e0.elapsed_time(e1)], world, dev)
        h2d = XKp.numel() * 2 * 2 + w.steps * (2 * w.B * w.Hkv * w.d + w.B * w.Hq * w.d) * 2
        d2h = w.steps * w.B * w.Hq * w.d * 4
        e2e = {"value": job_throughput(tokens_per_episode * args.steps, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / args.steps}

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, budget_s=20.0)

    peak, peak_kind = peaks()
    decode_launch_ms = decode_ms / (args.steps * w.steps)
    achieved = bytes_per_episode / w.steps / (decode_launch_ms / 1e3) / 1e9
    traffic = ncu_traffic(w)
    line = {
        "metric": METRIC,
        "value": job_throughput(tokens_per_episode * args.steps, world, ms),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"u{w.bits} codes, f32 accumulate",
        "data": "synthetic (seeded; distributions of the workload definition)",
        "config": {
            "workload": w.name, "batch_per_gpu": w.B, "global_batch": w.B * world,
            "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d, "prompt_tokens": w.T,
            "decode_steps": w.steps, "bits": w.bits, "group_k": w.G, "group_v": w.Gv,
            "residual": w.R, "symmetric": w.symmetric, "key_outliers_per_token": args.key_outliers,
            "elem": "fp16" if w.dtype == wl.FP16 else "bf16",
            "parallelism": f"dp{world} (independent sequences per GPU)",
            "l2": "inputs larger than L2: packed cache "
                  f"{bytes_per_episode / w.steps / 1e6:.0f} MB per decode step, prompt "
                  f"{2 * XK.numel() * 2 / 1e6:.0f} MB per step",
            "splits": cache.splits(),
            "timing": "value: K whole-episode CUDA-graph replays between two events; roofline: "
                      "events around every decode_attention graph in K more episodes replayed "
                      "step by step",
        },
        "decode_steps_per_s": w.steps * args.steps / (ms / 1e3),
        "kv_tokens_per_s_decode_only": job_throughput(tokens_per_episode * args.steps, world, decode_ms),
        "roofline": {
            "kernel": f"append + decode_attention ({decode_kernel_name(w)}: one launch without a flush, "
                      "splits merged in-kernel), per call",
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
            if peak_kind == "measured" else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_launch": bytes_per_episode / w.steps,
            "avg_launch_us": decode_launch_ms * 1e3,
            "traffic": traffic,
        },
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
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
                             f"decode_attention ({decode_kernel_name(w)}) over a LogQuant cache, per call")
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
                             f"paged decode_attention ({decode_kernel_name(w)}, paged instance), per call")
    _finish(world, rank, line)


# ---------------------------------------------------------------------------
# the CPU oracle (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def cpu_baseline(w, budget_s=20.0, steps=None):
    """Time the oracle (as it stands) on a bounded sample of the workload: one
    sequence (all of its kv heads), its prompt prefill and the first decode
    steps, stopping after ~budget_s seconds.  Returns KV tokens/s for that sample."""
    import oracle
    from bit_kv_cache_22_b200 import workloads as wl
    XK, XV = wl.prefill_bits(w, bs=[0])
    tK, tV, tQ = wl.decode_bits(w, bs=[0])
    t0 = time.perf_counter()
    c = oracle.OracleCache(1, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric, w.dtype)
    c.prefill(XK, XV)
    tokens, done = 0, 0
    limit = w.steps if steps is None else steps
    for s in range(limit):
        c.append(tK[s], tV[s])
        c.decode(tQ[s])
        tokens += c.Tq + c.r
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    return {"value": tokens / el, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"1 of {w.B} sequences (all {w.Hkv} kv heads): prefill of {w.T} tokens + "
                      f"{done} of {w.steps} decode steps, {el:.1f} s, fp64 C oracle with OpenMP"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from bit_kv_cache_22_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(w, budget_s=budget)
    vals = [cpu_baseline(w, budget_s=budget) for _ in range(args.steps)]
    v = statistics.mean(x["value"] for x in vals)
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "impl": "reference", "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": w.name, "global_batch": w.B, "note": "CPU oracle, rank 0"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": vals[0]["cores"],
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
