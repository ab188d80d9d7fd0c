"""include/q8.h is a plain C interface: a C11 program compiled with gcc
-Werror against it links libq8.so and gets the documented host-side
statuses (tests/c/abi_check.c; no device memory is touched)."""
import os
import shutil
import subprocess

import pytest

from bit_quantized_b200 import build as q8build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_consumer_compiles_links_and_validates():
    lib = q8build.build()
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, f"abi_check_{os.getpid()}")
    libdir = os.path.dirname(lib)
    cc = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror",
                         "-I" + os.path.join(ROOT, "include"),
                         os.path.join(ROOT, "tests", "c", "abi_check.c"),
                         "-L" + libdir, "-lq8", "-Wl,-rpath," + libdir, "-o", exe],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    try:
        run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    finally:
        os.remove(exe)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "FAIL" not in run.stdout and run.stdout.count("ok ") >= 7
