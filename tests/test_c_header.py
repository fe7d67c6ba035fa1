"""The boundary from plain C: include/kvq.h compiles as C11 with gcc, and a C program
linked against libkvq.so sizes a cache and plans a decode (host-only calls, no GPU)."""
import os
import subprocess
import tempfile

import pytest

from bit_kv_cache_22_b200 import kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "kvq.h"

int main(void) {
    kvq_config c = {8, 32, 32, 128, 128, 128, 128, 4, 0, KVQ_BF16, 4352};
    kvq_sizes s;
    if (kvq_get_sizes(&c, &s) != KVQ_OK) return 1;
    int64_t lengths[8];
    for (int i = 0; i < 8; ++i) lengths[i] = 4096 + 21;
    int32_t nq = 0, per = 0, S = 0;
    if (kvq_plan_decode(&c, lengths, 148, 4, &nq, &per, &S) != KVQ_OK) return 2;
    kvq_paged_config pc = {c, 128, 100};
    kvq_paged_sizes ps;
    if (kvq_paged_get_sizes(&pc, &ps) != KVQ_OK) return 3;
    c.bits = 3;
    if (kvq_get_sizes(&c, &s) != KVQ_ERR_UNSUPPORTED || kvq_last_error()[0] == 0) return 4;
    printf("%zu %d %d %d %zu %d\n", s.k_codes, nq, per, S, ps.page_table, kvq_layout_version());
    return 0;
}
"""


def test_header_compiles_as_c_and_links():
    lib = kvq.load()   # builds libkvq.so if needed
    del lib
    libdir = os.path.dirname(kvq.library_path())
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "abi.c")
        exe = os.path.join(d, "abi")
        with open(src, "w") as f:
            f.write(PROGRAM)
        cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o", exe,
               os.path.join(libdir, "libkvq.so"), f"-Wl,-rpath,{libdir}"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0 and "cannot find" in r.stderr:
            pytest.skip("the CUDA runtime the library links against is not on the linker path")
        assert r.returncode == 0, r.stderr
        out = subprocess.run([exe], capture_output=True, text=True)
        assert out.returncode == 0, (out.returncode, out.stderr)
        k_codes, nq, per, S, pt, layout = out.stdout.split()
        assert int(k_codes) == 8 * 32 * 4352 * 128 * 4 // 8      # sizes of the last valid config
        assert (int(nq), int(per), int(S)) == (2, 128, 3)      # 2 quantized splits + 1 residual split
        assert int(pt) == 8 * (4352 // 128) * 4 and int(layout) == 2
