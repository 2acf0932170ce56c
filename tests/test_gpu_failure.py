"""Failure detection without a GPU fault.

Every pipeline wait in the kernels is a bounded mbarrier wait: after its limit
it sets the CTA's abort flag, writes the device-timeout code to the caller's
error word and returns, so the kernel ends normally and the context stays
usable.  jl_wait_timeout_check runs that same wait on a barrier that nothing
completes (with a short limit): the error word must read 1, the call must end
after about the limit, and a decode launched right after must still match the
fp64 oracle.
"""

import time

import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic
from tests.gpu_helpers import assert_close, run_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_context_extension_b200 import build
    build.build()
    assert torch.cuda.is_available()


def test_bounded_wait_runs_out_reports_and_leaves_the_context_usable():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    jl.jl_wait_timeout_check(err, timeout_s=0.2)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(err.item()) == 1, "the starved wait must report the device-timeout code"
    assert 0.15 < dt < 5.0, dt

    # the same context runs a decode correctly right after
    B, L, Hq, Hkv, D, W, w0 = 1, 3000, 4, 1, 128, 1000, 200
    q, kc, vc = synthetic.decode_inputs(B, L, Hq, Hkv, D, seed=5)
    o, lse, derr = run_decode(q, kc, vc, L=L, w0=w0, W=W, base=1e6)
    assert derr == 0
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e6)
    o_ref, lse_ref = jo.decode(q.double().numpy(), kc.double().numpy(), vc.double().numpy(), p)
    assert_close(o.numpy(), o_ref, lse.numpy(), lse_ref, "decode after a timeout")
