"""The boundary from plain C on a GPU: a C11 program that allocates every device buffer
itself (cudaMalloc), creates a cache over them, prefills and decodes through include/kvq.h,
and checks that kvq_create takes no device memory of its own (cudaMemGetInfo unchanged),
that the output is finite and that the device status stays clear."""
import os
import subprocess
import tempfile

import pytest
import torch

from bit_kv_cache_22_b200 import kvq

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"

PROGRAM = r"""
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime_api.h>
#include "kvq.h"

#define CK(x) do { if ((x) != cudaSuccess) { printf("cuda error line %d\n", __LINE__); return 10; } } while (0)

int main(void) {
    kvq_config c = {2, 8, 2, 128, 32, 32, 128, 2, 0, KVQ_BF16, 1024};
    kvq_sizes s;
    if (kvq_get_sizes(&c, &s) != KVQ_OK) return 1;
    kvq_buffers b;
    CK(cudaMalloc(&b.k_codes, s.k_codes)); CK(cudaMalloc((void **)&b.k_scales, s.k_scales));
    CK(cudaMalloc((void **)&b.k_zeros, s.k_zeros)); CK(cudaMalloc(&b.v_codes, s.v_codes));
    CK(cudaMalloc((void **)&b.v_scales, s.v_scales)); CK(cudaMalloc((void **)&b.v_zeros, s.v_zeros));
    CK(cudaMalloc(&b.k_residual, s.k_residual)); CK(cudaMalloc(&b.v_residual, s.v_residual));
    CK(cudaMalloc(&b.state, s.state));
    void *ws; CK(cudaMalloc(&ws, s.workspace));
    const int T = 3 * 128 + 17;
    const size_t nx = (size_t)c.batch * c.kv_heads * T * c.head_dim;
    unsigned short *hx = (unsigned short *)malloc(nx * 2);
    srand(1);
    for (size_t i = 0; i < nx; ++i) {           /* bf16 patterns of values in [-2, 2) */
        float f = (float)rand() / RAND_MAX * 4.0f - 2.0f;
        unsigned int u; memcpy(&u, &f, 4); hx[i] = (unsigned short)(u >> 16);
    }
    void *xk, *xv, *q; float *o;
    CK(cudaMalloc(&xk, nx * 2)); CK(cudaMalloc(&xv, nx * 2));
    CK(cudaMemcpy(xk, hx, nx * 2, cudaMemcpyHostToDevice)); CK(cudaMemcpy(xv, hx, nx * 2, cudaMemcpyHostToDevice));
    const size_t nq = (size_t)c.batch * c.q_heads * c.head_dim;
    CK(cudaMalloc(&q, nq * 2)); CK(cudaMemcpy(q, hx, nq * 2, cudaMemcpyHostToDevice));
    CK(cudaMalloc((void **)&o, nq * 4));
    CK(cudaDeviceSynchronize());
    size_t free0, free1, total;
    CK(cudaMemGetInfo(&free0, &total));
    kvq_cache *h = NULL;
    if (kvq_create(&c, &b, &h) != KVQ_OK) { printf("%s\n", kvq_last_error()); return 2; }
    CK(cudaDeviceSynchronize());
    CK(cudaMemGetInfo(&free1, &total));
    if (free1 != free0) { printf("kvq_create took %zu bytes\n", free0 - free1); return 3; }
    if (kvq_prefill_quantize(h, xk, xv, T, NULL) != KVQ_OK) return 4;
    if (kvq_decode_attention(h, q, o, ws, s.workspace, NULL) != KVQ_OK) return 5;
    float *ho = (float *)malloc(nq * 4);
    CK(cudaMemcpy(ho, o, nq * 4, cudaMemcpyDeviceToHost));
    for (size_t i = 0; i < nq; ++i) if (!isfinite(ho[i])) return 6;
    if (kvq_check_device(h) != KVQ_OK) return 7;
    CK(cudaMemGetInfo(&free1, &total));
    kvq_destroy(h);
    printf("ok %zu\n", free0 - free1);
    return 0;
}
"""


def test_c_program_owns_every_buffer():
    kvq.load()
    libdir = os.path.dirname(kvq.library_path())
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "prog.c"), os.path.join(d, "prog")
        with open(src, "w") as f:
            f.write(PROGRAM)
        cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I",
               f"{CUDA}/include", src, "-o", exe, os.path.join(libdir, "libkvq.so"), f"-L{CUDA}/lib64",
               "-lcudart", "-lm", f"-Wl,-rpath,{libdir}:{CUDA}/lib64"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
        assert out.stdout.startswith("ok 0"), out.stdout     # no device memory taken by any call


def test_create_takes_no_device_memory_through_the_binding():
    from bit_kv_cache_22_b200 import workloads as wl
    import kvq_testlib as tl
    w = wl.WORKLOADS["gqa8b"].replace(B=2, Hkv=2, Hq=8, T=300, steps=1)
    a = tl.new_cache(w)                       # warms the library and the allocator up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    lib = kvq.load()
    import ctypes
    h = ctypes.c_void_p()
    bufs = kvq.Buffers(a.k_codes.data_ptr(), a.k_scales.data_ptr(), a.k_zeros.data_ptr(), a.v_codes.data_ptr(),
                       a.v_scales.data_ptr(), a.v_zeros.data_ptr(), a.k_residual.data_ptr(),
                       a.v_residual.data_ptr(), a.state_buf.data_ptr())
    assert lib.kvq_create(ctypes.byref(a.cfg), ctypes.byref(bufs), ctypes.byref(h)) == kvq.KVQ_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    lib.kvq_destroy(h)
