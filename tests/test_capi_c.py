"""The C ABI from C: tests/capi_consumer.c includes include/mea.h as a C99
translation unit (gcc -std=c99 -pedantic -Werror), links libmea.so and runs
validation-only calls, so it needs no GPU.  This checks that the header is a
plain C header (no C++ or CUDA types in the signatures) and that a C program
sees the same status codes as the Python binding."""
import os
import shutil
import subprocess

import pytest

from memory_efficient_activation_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "capi_consumer.c")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_consumer_compiles_links_and_runs(tmp_path):
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "capi_consumer")
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           SRC, "-o", exe, "-L", libdir, "-l:libmea.so", "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
