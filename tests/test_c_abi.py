"""The C ABI from plain C: include/kvq.h compiles as strict C99, and a C program linked
against libkvq.so runs the host-side entry points (planning, workspace sizes, argument
errors, the per-tag allocator) without a GPU."""
import os
import shutil
import subprocess

import pytest

from layer_wise_mixed_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_against_the_library(tmp_path):
    lib = build.build()
    exe = tmp_path / "c_abi_host"
    src = os.path.join(ROOT, "tests", "c_abi_host.c")
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"), src,
           "-L", libdir, "-lkvq", f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("all ok")
