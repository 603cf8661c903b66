"""Build the decoder's shared library in-tree with nvcc for sm_100a.

``python -m kv_cache_decode_dualcache_b200.build`` (or ``build()``) compiles
``csrc/*.cu`` into ``libfdllm.so`` next to this file.  Nothing is
JIT-compiled at import time; the binding loads the prebuilt library and fails
loudly when it is missing.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libfdllm.so")
# Self-checking variant: every device access of the GEMM / epilogue bounds-
# checked, violations recorded and reported as FDLLM_ERR_CUDA.
LIB_CHECKS = os.path.join(HERE, "libfdllm_checks.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libfdllm.so")


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh"))) + sorted(
        glob.glob(os.path.join(HERE, "csrc", "*.h"))) + [os.path.join(ROOT, "include", "fdllm.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False, extra=None, checks: bool = False) -> str:
    lib = LIB_CHECKS if checks else LIB
    if not force and up_to_date(lib):
        return lib
    nvcc = _nvcc()
    objdir = os.path.join(ROOT, "_build", "checks" if checks else "release")
    os.makedirs(objdir, exist_ok=True)
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler",
                    "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
                    "--expt-relaxed-constexpr"] + (["-DFDLLM_CHECKS"] if checks else []) + \
        list(extra or [])
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc, "-c", src, "-o", obj] + flags
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT), src))
        objs.append(obj)
    for p, src in procs:
        out, _ = p.communicate()
        if p.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{out.decode(errors='replace')}")
        if verbose and out:
            print(out.decode(errors="replace"), file=sys.stderr)
    tmp = lib + ".tmp"
    cmd = [nvcc, "-shared", "-o", tmp] + objs + ARCH + ["-Xcompiler", "-fPIC"]
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n" + r.stdout.decode(errors="replace"))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                checks="--checks" in sys.argv))
