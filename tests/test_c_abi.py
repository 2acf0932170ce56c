"""The boundary from plain C.

* tests/c/abi_smoke.c includes include/jl_api.h as strict C99 (-pedantic,
  warnings as errors), links libjetlong.so by path and calls the host-only
  entry points.  No GPU.
* tests/c/prefill_from_c.c (GPU; C11, since the CUDA runtime's headers are
  not strict C99) runs a prefill with device memory from the CUDA runtime and
  no Python in the process; its outputs are held to the fp64 oracle on the
  same seeded inputs.
"""

import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic

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


def _cuda_home():
    for cand in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if cand and os.path.exists(os.path.join(cand, "include", "cuda_runtime.h")):
            return cand
    return None


@pytest.mark.gpu
def test_prefill_from_a_c_program(tmp_path):
    cuda = _cuda_home()
    assert cuda is not None and shutil.which("gcc") is not None
    lib = jl.library_path
    exe = tmp_path / "prefill_from_c"
    # (C11: the CUDA runtime's own headers use anonymous unions)
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "prefill_from_c.c"), lib,
           f"-Wl,-rpath,{os.path.dirname(lib)}", "-L", os.path.join(cuda, "lib64"), "-lcudart",
           f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    B, L, Hq, Hkv, D, w0, W, base = 1, 700, 8, 2, 128, 150, 200, 10000.0  # G 4, ragged tiles
    q, k, v = synthetic.prefill_inputs(B, L, Hq, Hkv, D, seed=5)
    files = {n: tmp_path / f"{n}.bin" for n in ("q", "k", "v", "o", "lse")}
    for n, t in (("q", q), ("k", k), ("v", v)):
        t.contiguous().view(torch.int16).numpy().tofile(files[n])
    args = [str(x) for x in (B, L, Hq, Hkv, D, w0, W, base)] + [str(files[n]) for n in ("q", "k", "v", "o", "lse")]
    r = subprocess.run([str(exe), *args], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, f"step {r.returncode}: {r.stderr}"
    o = torch.from_numpy(np.fromfile(files["o"], dtype=np.int16)).view(torch.bfloat16).float().reshape(B, L, Hq, D)
    lse = np.fromfile(files["lse"], dtype=np.float32).reshape(B, Hq, L)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=base)
    o_ref, lse_ref = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    from tests.gpu_helpers import assert_close
    assert_close(o.numpy(), o_ref, lse, lse_ref, "prefill from C")
