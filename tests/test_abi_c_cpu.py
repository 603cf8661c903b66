"""The C ABI from a plain C program (no Python, no torch): compile
tests/abi_c/abi_smoke.c with gcc against include/fdllm.h, link it with
libfdllm.so and run the argument checks that need no GPU."""
import os
import shutil
import subprocess
import tempfile

import pytest

from kv_cache_decode_dualcache_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plain_c_caller_links_and_passes_the_argument_checks():
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc is not installed")
    lib = build.build()
    libdir = os.path.dirname(lib)
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "abi_smoke")
        cc = subprocess.run([gcc, "-std=c11", "-Wall", "-Werror",
                             "-I", os.path.join(ROOT, "include"),
                             os.path.join(ROOT, "tests", "abi_c", "abi_smoke.c"),
                             "-o", exe, lib, f"-Wl,-rpath,{libdir}", "-lm"],
                            capture_output=True, text=True, timeout=120)
        assert cc.returncode == 0, cc.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "abi_smoke ok"
