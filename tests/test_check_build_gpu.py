"""The bounds-check build (libkvq_check.so, selected by KVQ_LIBRARY=check) on a GPU.

* The parity suites pass under it: every index the kernels take from a list stays in
  its buffer (a bad one would raise status bit 3).
* A bounded wait made to run out -- on a shared-memory barrier that nothing arrives at --
  gives up: kvq_check_device reports KVQ_ERR_DEVICE_CHECK, and the same context then
  decodes correctly (no fault, no hang).
* An out-of-range row index handed to the gather kernel is reported and not followed.

Each case runs in a child process, since the library a process loads is fixed at its
first use.
"""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(code: str, timeout=600):
    env = dict(os.environ, KVQ_LIBRARY="check", PYTHONPATH=os.pathsep.join([ROOT, os.path.join(ROOT, "tests")]))
    r = subprocess.run([sys.executable, "-c", textwrap.dedent(code)], capture_output=True, text=True, env=env,
                       cwd=ROOT, timeout=timeout)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    return r.stdout


def test_parity_suites_under_the_bounds_check_build():
    env = dict(os.environ, KVQ_LIBRARY="check")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        "tests/test_parity_gpu.py", "tests/test_logquant_gpu.py", "tests/test_paged_gpu.py",
                        "tests/test_sparse_gpu.py"],
                       capture_output=True, text=True, env=env, cwd=ROOT, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:]
    assert " passed" in r.stdout


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    out = _run("""
        import numpy as np, torch
        from bit_kv_cache_22_b200 import kvq, workloads as wl
        import kvq_testlib as tl
        assert kvq.check_build() and kvq.library_path().endswith("libkvq_check.so")
        w = wl.WORKLOADS["gqa8b"].replace(B=2, Hkv=2, Hq=8, T=6 * 128 + 9, steps=2)
        XK, XV = wl.prefill_bits(w)
        tK, tV, tQ = wl.decode_bits(w)
        cache, ref = tl.new_cache(w), tl.new_oracle(w)
        cache.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
        ref.prefill(XK, XV)
        lib = kvq.load()
        assert lib.kvq_debug_set_stall(cache._h, 8) == kvq.KVQ_OK
        cache.decode_attention(tl.to_dev(tQ[0], w))
        torch.cuda.synchronize()
        try:
            cache.check_device()
            raise SystemExit("the wait did not give up")
        except kvq.KVQError as e:
            assert e.status == kvq.KVQ_ERR_DEVICE_CHECK, e
            assert b"gave up waiting" in lib.kvq_last_error()
        assert lib.kvq_debug_set_stall(cache._h, 0) == kvq.KVQ_OK
        cache.append(tl.to_dev(tK[0], w), tl.to_dev(tV[0], w))
        ref.append(tK[0], tV[0])
        got = cache.decode_attention(tl.to_dev(tQ[1], w)).cpu().numpy()
        tl.assert_close(got, ref.decode(tQ[1]), "after the stall")
        cache.check_device()
        print("ok")
    """)
    assert out.strip().endswith("ok")


def test_a_bad_gather_index_is_reported_not_followed():
    out = _run("""
        import numpy as np, torch
        from bit_kv_cache_22_b200 import kvq, workloads as wl
        import kvq_testlib as tl
        w = wl.WORKLOADS["gqa8b"].replace(B=1, Hkv=1, Hq=4, T=128, steps=1)
        cache = tl.new_cache(w)
        src = torch.arange(10 * w.d, dtype=torch.int16, device="cuda").view(10, w.d)
        dst = torch.zeros(4, w.d, dtype=torch.int16, device="cuda")
        idx = torch.tensor([0, 3, 12, 9], dtype=torch.int32, device="cuda")     # 12 is outside the 10 rows
        lib = kvq.load()
        s = torch.cuda.current_stream().cuda_stream
        assert lib.kvq_debug_gather_rows(cache._h, src.data_ptr(), 10, idx.data_ptr(), 4, dst.data_ptr(), s) == 0
        torch.cuda.synchronize()
        try:
            cache.check_device()
            raise SystemExit("the bad index was not reported")
        except kvq.KVQError as e:
            assert e.status == kvq.KVQ_ERR_DEVICE_CHECK, e
        assert torch.equal(dst[0], src[0]) and torch.equal(dst[1], src[3]) and torch.equal(dst[3], src[9])
        assert torch.equal(dst[2], src[0])                      # row 0 instead of the bad one
        idx = torch.tensor([1, 2, 3, 4], dtype=torch.int32, device="cuda")
        assert lib.kvq_debug_gather_rows(cache._h, src.data_ptr(), 10, idx.data_ptr(), 4, dst.data_ptr(), s) == 0
        cache.check_device()                                   # good indices raise nothing
        assert torch.equal(dst, src[1:5])
        print("ok")
    """)
    assert out.strip().endswith("ok")
