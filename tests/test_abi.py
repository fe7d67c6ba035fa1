"""The C ABI without a GPU: the library loads, exports what include/kvq.h declares,
and validates configurations on the host."""
import ctypes
import os
import re
import subprocess

import pytest

from bit_kv_cache_22_b200 import kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", text)))


def test_header_declares_the_three_operations():
    names = declared_symbols()
    for op in ("kvq_prefill_quantize", "kvq_append", "kvq_decode_attention"):
        assert op in names
    assert set(names) == set(kvq.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = kvq.load()
    out = subprocess.run(["nm", "-D", "--defined-only", kvq.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (kvq_\w+)", out))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(lib, name)
    # nothing else with the public prefix leaks out
    assert exported == set(declared_symbols())


def test_library_is_built_for_sm100a_only():
    from bit_kv_cache_22_b200 import build
    flags = build.NVCC_FLAGS
    targets = [flags[i + 1] for i, f in enumerate(flags) if f == "-gencode"]
    assert targets == ["arch=compute_100a,code=sm_100a"]


@pytest.mark.gpu
def test_loaded_kernels_are_sm100():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()
    assert kvq.load().kvq_binary_arch() == 100


def _cfg(**kw):
    base = dict(batch=1, q_heads=4, kv_heads=2, head_dim=128, group_k=32, group_v=32,
                residual=128, bits=2, symmetric=0, dtype=kvq.KVQ_BF16, capacity=1024)
    base.update(kw)
    return kvq.Config(**base)


def test_sizes_match_layout():
    s = kvq.get_sizes(_cfg())
    BH, cap, d = 2, 1024, 128
    assert s.k_codes == s.v_codes == BH * cap * d * 2 // 8
    assert s.k_scales == BH * (cap // 32) * d * 4 and s.k_zeros == BH * (cap // 32) * d * 2
    assert s.v_scales == BH * cap * (d // 32) * 4 and s.v_zeros == BH * cap * (d // 32) * 2
    assert s.k_residual == s.v_residual == BH * 128 * d * 2
    assert s.workspace > 0
    # state: a split-arrival counter per (batch, query head) and the status word, 16-byte padded
    assert s.state == -(-(1 * 4 + 1) * 4 // 16) * 16
    sym = kvq.get_sizes(_cfg(symmetric=1, bits=4))
    assert sym.k_zeros == 0 and sym.v_zeros == 0


def test_logquant_state_holds_the_row_lists():
    lib = kvq.load()
    cfg, W = _cfg(capacity=1536), 128
    s = kvq.Sizes()
    assert lib.kvq_logquant_get_sizes(ctypes.byref(cfg), W, ctypes.byref(s)) == kvq.KVQ_OK
    cap = -(-1536 // (3 * W)) * 3 * W
    assert s.state == 32 + (W + cap + 3 * W) * 4          # counters (5 words, padded) + lists


def test_create_needs_a_state_buffer():
    lib = kvq.load()
    cfg = _cfg()
    fake = 1 << 20                                 # aligned, never dereferenced: rejected first
    bufs = kvq.Buffers(*([fake] * 8), None)
    h = ctypes.c_void_p()
    assert lib.kvq_create(ctypes.byref(cfg), ctypes.byref(bufs), ctypes.byref(h)) == kvq.KVQ_ERR_INVALID_ARG
    assert b"state" in lib.kvq_last_error() and not h.value
    bufs = kvq.Buffers(*([fake] * 8), fake + 8)    # misaligned state
    assert lib.kvq_create(ctypes.byref(cfg), ctypes.byref(bufs), ctypes.byref(h)) == kvq.KVQ_ERR_INVALID_ARG


@pytest.mark.parametrize("bad,status", [
    (dict(head_dim=96), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(bits=3), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(q_heads=3), kvq.KVQ_ERR_INVALID_ARG),
    (dict(group_k=24), kvq.KVQ_ERR_INVALID_ARG),
    (dict(group_k=48, residual=96), kvq.KVQ_ERR_INVALID_ARG),
    (dict(group_v=48), kvq.KVQ_ERR_INVALID_ARG),
    (dict(residual=48), kvq.KVQ_ERR_INVALID_ARG),
    (dict(capacity=1000), kvq.KVQ_ERR_INVALID_ARG),
    (dict(dtype=7), kvq.KVQ_ERR_INVALID_ARG),
    (dict(batch=0), kvq.KVQ_ERR_INVALID_ARG),
    (dict(group_v=256, head_dim=128), kvq.KVQ_ERR_INVALID_ARG),
])
def test_invalid_configs_are_rejected(bad, status):
    with pytest.raises(kvq.KVQError) as ei:
        kvq.get_sizes(_cfg(**bad))
    assert ei.value.status == status
    assert kvq.load().kvq_last_error()


def test_null_arguments_are_rejected_without_a_device():
    lib = kvq.load()
    assert lib.kvq_get_sizes(None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_prefill_quantize(None, None, None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_append(None, None, None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_decode_attention(None, None, None, None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_decode_splits(None) == 0
    assert lib.kvq_check_device(None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_append_decode_attention(None, None, None, None, None, None, 0, None) == \
        kvq.KVQ_ERR_INVALID_ARG
    lib.kvq_destroy(None)
    h = ctypes.c_void_p()
    cfg = _cfg()
    bufs = kvq.Buffers()
    assert lib.kvq_create(ctypes.byref(cfg), ctypes.byref(bufs), ctypes.byref(h)) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert not h.value
    assert lib.kvq_layout_version() == 2


def _paged(page_tokens=128, num_pages=10, **kw):
    return kvq.PagedConfig(_cfg(**kw), page_tokens, num_pages)


def test_paged_sizes_match_layout():
    lib = kvq.load()
    s = kvq.PagedSizes()
    assert lib.kvq_paged_get_sizes(ctypes.byref(_paged()), ctypes.byref(s)) == kvq.KVQ_OK
    slices, P, d = 10 * 2, 128, 128                 # num_pages * kv_heads
    assert s.k_codes == s.v_codes == slices * P * d * 2 // 8
    assert s.k_scales == slices * (P // 32) * d * 4 and s.k_zeros == slices * (P // 32) * d * 2
    assert s.v_scales == slices * P * (d // 32) * 4 and s.v_zeros == slices * P * (d // 32) * 2
    assert s.k_residual == s.v_residual == 2 * 128 * d * 2
    assert s.page_table == 1 * (1024 // 128) * 4
    assert s.workspace == kvq.get_sizes(_cfg()).workspace
    assert s.state == kvq.get_sizes(_cfg()).state + 16      # + the slots' lengths, padded


@pytest.mark.parametrize("bad", [dict(page_tokens=96), dict(page_tokens=64),   # not a multiple of R = 128
                                 dict(page_tokens=384), dict(num_pages=0),     # capacity 1024 % 384
                                 dict(page_tokens=0), dict(head_dim=96)])
def test_invalid_paged_configs_are_rejected(bad):
    lib = kvq.load()
    P = bad.pop("page_tokens", 128)
    n = bad.pop("num_pages", 10)
    s = kvq.PagedSizes()
    assert lib.kvq_paged_get_sizes(ctypes.byref(_paged(P, n, **bad)), ctypes.byref(s)) != kvq.KVQ_OK
    assert lib.kvq_last_error()


def test_paged_null_arguments_are_rejected_without_a_device():
    lib = kvq.load()
    assert lib.kvq_paged_get_sizes(None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_paged_prefill(None, 0, None, None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_paged_append(None, None, None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_paged_decode_attention(None, None, None, None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_paged_release(None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_paged_seq_len(None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_paged_check_device(None) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_paged_decode_splits(None) == 0
    lib.kvq_paged_destroy(None)
    h = ctypes.c_void_p()
    bufs = kvq.Buffers()
    assert lib.kvq_paged_create(ctypes.byref(_paged()), ctypes.byref(bufs), None, ctypes.byref(h)) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert not h.value
