"""Build ``libkvq.so`` (the CUDA library behind include/kvq.h) in-tree with nvcc for sm_100a.

``python -m bit_kv_cache_22_b200.build`` rebuilds when a source is newer than
the library.  No compatibility layers: one target, sm_100a.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libkvq.so")
# the bounds-check build (-DKVQ_CHECK): kernels check list indices, tests can make bounded waits
# give up (include/kvq_check.h)
LIB_CHECK = os.path.join(PKG, "libkvq_check.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    """Compile every translation unit (in parallel) and link libkvq.so (libkvq_check.so with
    check=True: the bounds-check build)."""
    lib = LIB_CHECK if check else LIB
    if not force and not _stale(lib):
        return lib
    flags = NVCC_FLAGS + (["-DKVQ_CHECK"] if check else [])
    objdir = os.path.join(PKG, "_build_check" if check else "_build")
    os.makedirs(objdir, exist_ok=True)
    tag = os.getpid()
    procs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + f".{tag}.o")
        cmd = [NVCC, *flags, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((subprocess.Popen(cmd), obj))
    failed = [p.args for p, _ in procs if p.wait() != 0]
    objs = [o for _, o in procs]
    try:
        if failed:
            raise subprocess.CalledProcessError(1, failed[0])
        tmp = lib + f".tmp{tag}"
        subprocess.run([NVCC, *flags, "-shared", "-o", tmp, *objs], check=True)
        os.replace(tmp, lib)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, check="--check" in sys.argv))
