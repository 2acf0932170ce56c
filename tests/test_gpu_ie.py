"""The pages' inclusion-exclusion prefill (three calls + merge) on the GPU.

Checks the unfused three-call formulation (Jet-Long review, "Method") against
the fp64 oracle at the standard tolerances on inputs without outliers.  On
inputs with x8 outlier keys the merge's W_B O_B - W_C O_C subtraction
amplifies each partial result's rounding by
kappa = (W_A + W_B + W_C) / (W_A + W_B - W_C), which has no bound when a key
inside the window dominates both B and C: there the test holds every row's
error to that amplification of the partials' error instead (the
formulation's documented failure), and holds the fused kernel, which selects
one score set per pair and subtracts nothing, to the standard tolerances on
the same inputs.
"""

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic
from tests.gpu_helpers import O_MAX_ABS, assert_close, run_prefill

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
                                             (777, 3, 1, 64, 200, 77), (640, 2, 2, 128, 100, 0),
                                             (1300, 8, 2, 128, 260, 100)])
def test_ie_matches_oracle(L, Hq, Hkv, D, W, w0):
    q, k, v = synthetic.prefill_inputs(1, L, Hq, Hkv, D, seed=L)
    o, lse = run_ie(q, k, v, w0=w0, W=W, base=1e4)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e4)
    o_ref, lse_ref = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    assert_close(o.numpy(), o_ref, lse.numpy(), lse_ref, f"ie L{L} w0{w0}")


def test_ie_error_on_outlier_keys_is_the_merge_amplification():
    L, Hq, Hkv, D, W, w0 = 1300, 8, 2, 128, 260, 100
    q, k, v = synthetic.prefill_inputs(1, L, Hq, Hkv, D, seed=77, outlier_frac=0.01)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e4)
    o_ref, lse_ref = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    o_ie, _ = run_ie(q, k, v, w0=w0, W=W, base=1e4)
    o_fu, l_fu, err = run_prefill(q, k, v, w0=w0, W=W, base=1e4)
    assert err == 0
    assert_close(o_fu.numpy(), o_ref, l_fu.numpy(), lse_ref, "fused kernel on outliers")
    rows = np.arange(L)
    kappa_max, worst = 0.0, 0.0
    for h in range(Hq):
        g = h // (Hq // Hkv)
        (_, la), (_, lb), (_, lc) = jo.inclusion_exclusion_parts(
            q[0, :, h].double().numpy(), rows, k[0, :, g].double().numpy(), v[0, :, g].double().numpy(), p)
        mm = np.maximum(np.maximum(la, lb), lc)
        wa, wb, wc = np.exp(la - mm), np.exp(lb - mm), np.exp(lc - mm)
        kappa = (wa + wb + wc) / (wa + wb - wc)
        e_row = np.abs(o_ie[0, :, h].numpy() - o_ref[0, :, h]).max(axis=1)
        # each partial carries at most the fused kernel's output error bound;
        # the merge multiplies it by kappa (plus the final bf16 rounding)
        assert np.all(e_row <= O_MAX_ABS * kappa + O_MAX_ABS), (h, float((e_row / kappa).max()))
        kappa_max = max(kappa_max, float(kappa.max()))
        worst = max(worst, float(e_row.max()))
    e_fu = np.abs(o_fu.numpy() - o_ref)
    print(f"outlier keys: fused O max error {e_fu.max():.3e}; three-call merge O max error {worst:.3e} "
          f"at merge amplification up to {kappa_max:.1f}")
    assert kappa_max > 10.0  # the workload does reach the cancelling regime
