"""The boundary is a C ABI: a plain C11 program (tests/c_client.c) compiled with gcc against
include/jmoe.h, linked with libjmoe.so, runs its host-decided calls (sizes, argument errors, T = 0)
on the CPU.  This checks that the header is valid C, not only C++, and that the library needs no
Python or torch to be used."""
import os
import shutil
import subprocess

import pytest

from int8_expert_weight_b200 import build as jbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_client_builds_and_runs(tmp_path):
    lib = jbuild.build()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "c_client"
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_client.c"), "-o", str(exe), lib, f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "c client ok"
