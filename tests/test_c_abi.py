"""The boundary from plain C: tests/c/abi_smoke.c includes include/jl_api.h as
strict C99 (-pedantic, warnings as errors), links libjetlong.so by path and
calls the host-only entry points.  No GPU."""

import os
import shutil
import subprocess

import pytest

from rope_context_extension_b200 import jetlong as jl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_program_links_and_calls_the_abi(tmp_path):
    lib = jl.library_path
    assert os.path.exists(lib), "build the library first (rope_context_extension_b200.build)"
    exe = tmp_path / "abi_smoke"
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_smoke.c"), lib, f"-Wl,-rpath,{os.path.dirname(lib)}",
           "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, f"check {r.returncode} failed: {r.stderr}"
    assert r.stdout.strip() == "device pointer not 16-byte aligned"
