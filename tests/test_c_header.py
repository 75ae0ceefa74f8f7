"""The boundary is a C ABI: include/fa.h compiles as C99 (no C++ types), and
a plain C program links against libfa.so and gets the documented results
from calls that return before any GPU work."""
import os
import shutil
import subprocess

import pytest

from exact_tiled_attention_31_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c99_client_compiles_links_and_runs(tmp_path):
    lib = build.build_library()
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", str(exe), "-L", os.path.dirname(lib), "-lfa",
           "-Wl,-rpath," + os.path.dirname(lib)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "FAIL" not in run.stdout and run.stdout.count("ok ") >= 12, run.stdout
