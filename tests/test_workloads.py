"""The seeded synthetic inputs: shapes, determinism and the stated distributions."""
import numpy as np
import torch

from bit_kv_cache_22_b200 import workloads as wl


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 100
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wl.to_bits(x, wl.BF16), ref)
    assert np.array_equal(wl.from_bits(ref, wl.BF16),
                          torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_slices_are_deterministic_and_independent():
    w = wl.WORKLOADS["gqa8b"]
    a = wl.prefill_slice(w, 3, 5, T=64)
    b = wl.prefill_slice(w, 3, 5, T=64)
    c = wl.prefill_slice(w, 3, 6, T=64)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.array_equal(a[0], c[0])


def test_outlier_channels_and_sink():
    w = wl.WORKLOADS["llama7b"]
    for h in range(3):
        ch = wl.outlier_channels(w, h)
        assert len(ch) == 4 and len(set(ch.tolist())) == 4
        k, v = wl.prefill_slice(w, 0, h, T=2048)
        std = k.std(axis=0)
        assert np.all(std[ch] > 6) and np.delete(std, ch).max() < 1.3
    w = wl.WORKLOADS["long131k"]
    k, v = wl.prefill_slice(w, 0, 0, T=512)
    assert np.abs(k[:4]).mean() > 10 and np.abs(k[4:]).mean() < 1
    w = wl.WORKLOADS["gqa8b"]
    k, v = wl.prefill_slice(w, 0, 0, T=2048)
    assert abs(v.std() - 0.5) < 0.02 and len(wl.outlier_channels(w, 0)) == 1


def test_decode_bits_head_mapping():
    w = wl.WORKLOADS["tiny"]
    tK, tV, tQ = wl.decode_bits(w)
    assert tK.shape == (w.steps, w.B, w.Hkv, w.d) and tQ.shape == (w.steps, w.B, w.Hq, w.d)
    # tiny appends plain N(0,1) tokens: no outlier channel in decode keys
    k, _ = wl.decode_slice(w.replace(steps=4096), 0, 0)
    assert k.std(axis=0).max() < 1.2


def test_ragged_lengths_are_seeded_and_in_range():
    spec = wl.RAGGED["ragged_gqa"]
    w = spec["base"]
    a = wl.ragged_lengths(w, spec["lo"], spec["hi"])
    assert a == wl.ragged_lengths(w, spec["lo"], spec["hi"])
    assert len(a) == w.B and all(spec["lo"] <= x <= spec["hi"] for x in a)
    assert a != wl.ragged_lengths(w.replace(seed=w.seed + 1), spec["lo"], spec["hi"])
    assert spec["page_tokens"] % w.R == 0 and spec["page_tokens"] % 64 == 0
