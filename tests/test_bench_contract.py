"""bench.py's host-side arithmetic and JSON contract, on CPU: the algorithmic bytes of a
decode call (the roofline's numerator) restated from the storage layout, the episode's
(Tq, r) sequence, and the keys of a decode-only line."""
import bench
from bit_kv_cache_22_b200 import workloads as wl


def test_algorithmic_bytes_per_token_and_head():
    # codes 2 d n / 8 + key scales/zeros d 6 / G + value scales/zeros (d / Gv) 6
    w = wl.WORKLOADS["llama7b"]
    per_tok = 2 * 128 * 4 // 8 + 128 * 6 // 128 + (128 // 128) * 6          # 140 B
    q_out = w.B * w.Hq * w.d * (2 + 4)
    assert per_tok == 140
    assert bench.algorithmic_bytes(w, 4096, 0) == w.B * w.Hkv * 4096 * per_tok + q_out
    # residual rows: K and V in e (2 bytes each)
    assert bench.algorithmic_bytes(w, 4096, 5) - bench.algorithmic_bytes(w, 4096, 0) == w.B * w.Hkv * 5 * 2 * w.d * 2
    g = wl.WORKLOADS["gqa8b"]
    assert bench.algorithmic_bytes(g, 128, 0) == g.B * g.Hkv * 128 * 112 + g.B * g.Hq * g.d * 6   # 112 B
    s = wl.WORKLOADS["stream4sym"]                                                # symmetric: 4 B of meta
    assert bench.algorithmic_bytes(s, 128, 0) == s.B * s.Hkv * 128 * 160 + s.B * s.Hq * s.d * 6


def test_episode_contexts_flush_at_the_last_step():
    w = wl.WORKLOADS["llama7b"]
    ctx = bench.episode_contexts(w)
    assert len(ctx) == w.steps and ctx[0] == (4096, 1) and ctx[-2] == (4096, 127)
    assert ctx[-1] == (4096 + 128, 0)                 # the 128th append flushes


class _Clock:
    def summary(self):
        return {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}


class _Args:
    steps, warmup = 4, 3


def test_decode_only_line_keys():
    w = wl.WORKLOADS["gqa8b"]
    line = bench._decode_only_line(_Args(), w, 1, 10.0, 10.0, 10 ** 9, 2 * 10 ** 9, 256, _Clock(),
                                   {"workload": "x"}, "k")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches", "clocks"):
        assert key in line, key
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    assert abs(line["value"] - 10 ** 9 / 0.010) < 1e-3                # tokens over the slowest rank's time
    assert line["config"]["workload"] == "x" and "l2" in line["config"]


def test_cpu_baseline_reports_model_cores_and_one_core():
    w = wl.WORKLOADS["tiny"].replace(steps=2)
    r = bench.cpu_baseline(w, budget_s=0.5, one_core_s=0.2)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
    assert r["cpu_model"] and r["host_cores"] >= 1
    assert r["one_core"]["cores"] == 1 and r["one_core"]["value"] > 0
    import oracle
    assert oracle.num_threads() == r["cores"]          # the thread count is restored


def test_decode_kernel_names_follow_the_library_choice():
    gqa, llama = wl.WORKLOADS["gqa8b"], wl.WORKLOADS["llama7b"]
    assert bench.decode_kernel_name(gqa) == "decode_mma_kernel"
    assert bench.decode_kernel_name(llama) == "decode_mma_kernel"
    assert bench.decode_kernel_name(gqa, paged=True) == "decode_tc_kernel"
    assert bench.decode_kernel_name(gqa, key_outliers=1) == "decode_tc_kernel"
    assert bench.decode_kernel_name(gqa.replace(Hq=64)) == "decode_split_kernel"    # 8 query heads per kv head
    for name, (value, kernel) in bench.DECODE_KERNELS.items():
        assert bench.decode_kernel_name(gqa, forced=name) == (kernel or "decode_mma_kernel")
    assert [v for v, _ in bench.DECODE_KERNELS.values()] == [0, 1, 2, 3]   # kvq_set_decode_kernel's values


def test_profile_traffic_is_read_only_for_the_current_source(tmp_path, monkeypatch):
    w = wl.WORKLOADS["gqa8b"]
    h = bench.kernel_source_hash("decode_mma_kernel")
    (tmp_path / "profiles").mkdir()
    f = tmp_path / "profiles" / "decode_mma_kernel_gqa8b.md"
    f.write_text(f"kernel source sha256[:16]: {h}\ndram bytes per launch: 1234\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: h)
    assert bench.ncu_traffic(w) == 1234
    f.write_text("kernel source sha256[:16]: 0000000000000000\ndram bytes per launch: 1234\n")
    assert bench.ncu_traffic(w) is None
