"""The C ABI from plain C: tests/abi_c_check.c is compiled as C99 (warnings
as errors) against include/attn.h, linked to the in-tree library and run.
It makes host-side calls and argument-error calls only, so it needs no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_abi_from_plain_c(tmp_path):
    from exact_io_aware_sm_b200 import build
    lib = build.build()
    exe = str(tmp_path / "abi_c_check")
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "abi_c_check.c"), "-L", libdir, "-lattn_b200", f"-Wl,-rpath,{libdir}",
           "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
