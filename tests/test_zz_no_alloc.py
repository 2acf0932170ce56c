"""The decode entry point that allocates nothing, checked on the GPU.

jl_bifocal_decode_noalloc exists for callers that cannot allocate device
memory (for example a plugin whose host framework owns every byte of device
memory in its own pool): its scratch is a fixed array inside the library.
This test calls it through the C ABI twice in a row, with different problem
sizes so the second call starts from the first one's leftovers in the shared
array, and compares each result with jl_bifocal_decode (caller workspace) on
the same inputs, within the parity tolerances of the other GPU tests.  The
file name makes pytest collect it last.
"""

import pytest
import torch

from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic

pytestmark = pytest.mark.gpu

O_MAX_ABS = 2e-2
LSE_MAX_ABS = 1e-3


def _workspace_decode(q, kc, vc, L, w0, W):
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    ws = torch.zeros(jl.jl_decode_workspace_bytes(B, L, Hq, Hkv, D), dtype=torch.uint8, device=q.device)
    jl.jl_bifocal_decode(q, kc, vc, o, lse, L=L, w0=w0, w_pretrained=W, rope_base=1e6, workspace=ws)
    return o, lse


def _noalloc_decode(q, kc, vc, L, w0, W, err):
    B, Hq, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    jl.jl_bifocal_decode_noalloc(q, kc, vc, o, lse, L=L, w0=w0, w_pretrained=W, rope_base=1e6, dev_error=err)
    return o, lse


def test_noalloc_decode_matches_workspace_decode_on_two_calls_in_a_row():
    from rope_context_extension_b200 import build
    build.build()
    dev = torch.device("cuda")
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    calls = [
        # B, Lmax, L, Hq, Hkv, D, W, w0, outliers
        (2, 6000, 5000, 8, 2, 128, 1300, 700, 0.01),
        (3, 4096, 4096, 16, 2, 64, 1000, 0, 0.0),
    ]
    for B, Lmax, L, Hq, Hkv, D, W, w0, outl in calls:
        q, kc, vc = synthetic.decode_inputs(B, Lmax, Hq, Hkv, D, seed=L, outlier_frac=outl, length=L)
        q, kc, vc = q.to(dev), kc.to(dev), vc.to(dev)
        o_ref, l_ref = _workspace_decode(q, kc, vc, L, w0, W)
        o_na, l_na = _noalloc_decode(q, kc, vc, L, w0, W, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.isfinite(o_na.float()).all() and torch.isfinite(l_na).all()
        assert (o_na.float() - o_ref.float()).abs().max().item() <= O_MAX_ABS
        assert (l_na - l_ref).abs().max().item() <= LSE_MAX_ABS


def test_noalloc_decode_rejects_problems_beyond_its_fixed_scratch():
    # 4096 sequences x 8 KV heads x 8 query heads each need far more than 4 MiB of partials.
    dev = torch.device("cuda")
    q = torch.zeros(4096, 64, 128, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(4096, 64, 8, 128, dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    with pytest.raises(jl.JetLongError) as exc:
        jl.jl_bifocal_decode_noalloc(q, kc, kc, o, None, L=64, w0=8, w_pretrained=16, rope_base=1e6)
    assert exc.value.status == -4  # JL_ERR_WORKSPACE
