"""The pages' inclusion-exclusion prefill (three calls + merge) on the GPU.

Checks the unfused three-call formulation (Jet-Long review, "Method") against
the fp64 oracle, and compares its error with the fused per-tile kernel on
inputs with x8 outlier keys, where the merge's W_B O_B - W_C O_C subtraction
amplifies the bf16 rounding of the partial outputs.
"""

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic
from tests.gpu_helpers import assert_close, run_prefill

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_context_extension_b200 import build
    build.build()


def run_ie(q, k, v, *, w0, W, base, mode=jl.JL_QSHIFT_SELF_EXTEND):
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o = torch.empty_like(qd)
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=DEV)
    ws = torch.empty(jl.jl_prefill_ie_workspace_bytes(B, L, Hq, Hkv, D, mode), dtype=torch.uint8, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    jl.jl_bifocal_prefill_ie(qd, kd, vd, o, lse, w0=w0, w_pretrained=W, rope_base=base, mode=mode, workspace=ws,
                             dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return o.float().cpu(), lse.cpu()


@pytest.mark.parametrize("L,Hq,Hkv,D,W,w0", [(512, 2, 1, 64, 128, 32), (1000, 4, 2, 128, 300, 200),
                                             (777, 3, 1, 64, 200, 77), (640, 2, 2, 128, 100, 0)])
def test_ie_matches_oracle(L, Hq, Hkv, D, W, w0):
    q, k, v = synthetic.prefill_inputs(1, L, Hq, Hkv, D, seed=L)
    o, lse = run_ie(q, k, v, w0=w0, W=W, base=1e4)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e4)
    o_ref, lse_ref = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    assert_close(o.numpy(), o_ref, lse.numpy(), lse_ref, f"ie L{L} w0{w0}", lse_tol=1e-2)


def test_ie_error_versus_fused_on_outlier_keys():
    # Same inputs, both GPU paths against the fp64 oracle.  The fused kernel
    # selects one score set per pair; the merge subtracts two bf16 partial
    # outputs.  Record both; the fused path must not be the less accurate one
    # by more than rounding noise.
    L, Hq, Hkv, D, W, w0 = 1300, 8, 2, 128, 260, 100
    q, k, v = synthetic.prefill_inputs(1, L, Hq, Hkv, D, seed=77, outlier_frac=0.01)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e4)
    o_ref, lse_ref = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    o_ie, l_ie = run_ie(q, k, v, w0=w0, W=W, base=1e4, mode=jl.JL_QSHIFT_SELF_EXTEND | jl.JL_REMOTE_SPLIT)
    o_fu, l_fu, err = run_prefill(q, k, v, w0=w0, W=W, base=1e4, split=True)
    assert err == 0
    e_ie = np.abs(o_ie.numpy() - o_ref)
    e_fu = np.abs(o_fu.numpy() - o_ref)
    print(f"O mean abs error: fused {e_fu.mean():.3e}, inclusion-exclusion {e_ie.mean():.3e}; "
          f"max: fused {e_fu.max():.3e}, inclusion-exclusion {e_ie.max():.3e}")
    assert e_fu.mean() <= 1.05 * e_ie.mean()
    assert_close(o_fu.numpy(), o_ref, l_fu.numpy(), lse_ref, "fused split on outliers")
