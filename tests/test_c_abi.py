"""The boundary is a C ABI: a plain C program compiled with gcc against
include/fa.h and linked to libfa.so calls the entry points and gets the
documented status codes (validation paths only; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

import tiled_attention_20_b200.build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_calls_the_abi(tmp_path):
    lib = fa_build.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "abi_from_c")
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-o", exe,
                           os.path.join(ROOT, "tests", "c", "abi_from_c.c"),
                           "-I", os.path.join(ROOT, "include"),
                           "-L", libdir, "-l:" + os.path.basename(lib),
                           "-Wl,-rpath," + libdir])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("OK")
