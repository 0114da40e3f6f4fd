"""The boundary is a C ABI: a plain C11 program including include/bitlinear.h
compiles with gcc, links against libbitlinear.so and runs its host-only
calls (no GPU needed)."""

import os
import shutil
import subprocess

import pytest

from bitlinear_bl_forward_b200 import build as blbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_include():
    for cand in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        inc = os.path.join(cand, "include")
        if cand and os.path.exists(os.path.join(inc, "cuda_runtime_api.h")):
            return inc
    return None


def test_header_is_plain_c_and_links(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    inc = _cuda_include()
    if cc is None or inc is None:
        pytest.skip("needs a C compiler and the CUDA headers")
    blbuild.build()
    libdir = os.path.dirname(blbuild.LIB)
    exe = str(tmp_path / "c_abi_check")
    cmd = [cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           "-I", inc, os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe,
           "-L", libdir, "-lbitlinear", "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi check: ok" in r.stdout
