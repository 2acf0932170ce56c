"""The FMA-pipe exponential of the prefill softmax against CUDA's exp2f.

Prefill computes one pair of exponentials in every four with Cody-Waite range
reduction and a fitted degree-3 polynomial (csrc/exp2_poly_fit.py, max relative
error 8.6e-5 by construction).  Checked on the device over the range the
softmax produces, x in [-127, 8] (the lazy rescale keeps x <= 8), plus the
exact points: integers and the flush to 0 at and below -127.
"""

import numpy as np
import pytest
import torch

from rope_context_extension_b200 import jetlong as jl

pytestmark = pytest.mark.gpu


def test_exp2_polynomial_against_cuda_exp2f():
    from rope_context_extension_b200 import build
    build.build()
    x = torch.linspace(-126.0, 8.0, 2_000_001, dtype=torch.float32, device="cuda")
    yp, yr = jl.jl_exp2_poly_check(x)
    torch.cuda.synchronize()
    rel = ((yp.double() - yr.double()).abs() / yr.double()).max().item()
    assert rel <= 1.0e-4, rel
    xi = torch.arange(-126, 9, dtype=torch.float32, device="cuda")
    yp, yr = jl.jl_exp2_poly_check(xi)
    assert torch.equal(yp, yr)                      # exact at integers
    xz = torch.tensor([-127.0, -130.0, -1e30, float("-inf")], device="cuda")
    yp, _ = jl.jl_exp2_poly_check(xz)
    assert torch.equal(yp, torch.zeros_like(yp))     # flushed to zero like ex2.approx.ftz
