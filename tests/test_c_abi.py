"""The C ABI from plain C: tests/c/abi_probe.c is compiled as C99 with
warnings as errors against include/fa_b200.h, linked against libfa_b200.so
and run.  It makes only calls that fail an argument check, so it launches
nothing and runs the same on a machine with or without a GPU."""
import os
import shutil
import subprocess

import pytest

from flashattention_bf16_fwd_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_c_program_calls_every_entry_point(tmp_path):
    lib = fa_build.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "abi_probe")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_probe.c"),
           "-L", libdir, "-lfa_b200", f"-Wl,-rpath,{libdir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr
