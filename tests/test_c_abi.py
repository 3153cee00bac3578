"""The boundary is a C ABI: a plain C99 program compiles against
include/knapspec.h alone (-Wall -Werror), links libknapspec.so and runs its
host-only calls.  No GPU needed."""
import os
import shutil
import subprocess

import pytest

from knapsack_layer_selection_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_uses_the_abi(tmp_path):
    lib = BUILD.build()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "abi_host_check"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host_check.c"),
                    "-L", libdir, "-l:libknapspec.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "FAIL" not in out.stdout and out.stdout.count("ok ") == 8
