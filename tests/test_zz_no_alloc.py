"""The decode entry point that allocates nothing, checked on the GPU.

jl_bifocal_decode_noalloc exists for callers that cannot allocate device
memory (for example a plugin whose host framework owns every byte of device
memory in its own pool, or a serving loop that must not allocate once it
runs): its scratch is a fixed array inside the library.  These tests call it
through the C ABI several times in a row, with different problem sizes so each
call starts from the previous one's leftovers in the shared array, and compare
each result with jl_bifocal_decode (caller workspace) on the same inputs: bit
for bit where both use the same split count (same kernel, same inputs), within
the parity tolerances where the fixed array forces fewer splits, and always
against the fp64 oracle.  The file name makes pytest collect it last.
"""

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic

pytestmark = pytest.mark.gpu

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
FIXED_SCRATCH_BYTES = 4 << 20


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


def _against_oracle(q, kc, vc, o, lse, L, w0, W, what):
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e6)
    o_ref, lse_ref = jo.decode(q.float().cpu().numpy(), kc.float().cpu().numpy(), vc.float().cpu().numpy(), p)
    e = np.abs(o.float().cpu().numpy() - o_ref)
    le = np.abs(lse.cpu().numpy() - lse_ref)
    assert e.max() <= O_MAX_ABS and e.mean() <= O_MEAN_ABS and le.max() <= LSE_MAX_ABS, (what, e.max(), le.max())


# B, Lmax, L, Hq, Hkv, D, W, w0, outliers
SAME_SPLITS = [
    (2, 6000, 5000, 8, 2, 128, 1300, 700, 0.01),
    (3, 4096, 4096, 16, 2, 64, 1000, 0, 0.0),
    (1, 64, 64, 64, 8, 128, 16, 8, 0.0),          # GQA 8, D 128, B 1 (a short cache)
    (1, 131072, 131072, 64, 8, 128, 32768, 4096, 0.01),  # GQA 8, D 128, B 1, the 128K length
]


def test_noalloc_decode_equals_workspace_decode_on_calls_in_a_row():
    from rope_context_extension_b200 import build
    build.build()
    dev = torch.device("cuda")
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for B, Lmax, L, Hq, Hkv, D, W, w0, outl in SAME_SPLITS:
        q, kc, vc = synthetic.decode_inputs(B, Lmax, Hq, Hkv, D, seed=L, outlier_frac=outl, length=L)
        q, kc, vc = q.to(dev), kc.to(dev), vc.to(dev)
        o_ref, l_ref = _workspace_decode(q, kc, vc, L, w0, W)
        o_na, l_na = _noalloc_decode(q, kc, vc, L, w0, W, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        # same kernel, inputs and split count: the same bits
        assert torch.equal(o_na, o_ref) and torch.equal(l_na, l_ref), (B, L, Hq, Hkv, D)
        if B * Hq * L <= 64 * 131072:
            _against_oracle(q, kc, vc, o_na, l_na, L, w0, W, f"noalloc B{B} L{L}")
        del q, kc, vc


def test_noalloc_decode_with_fewer_splits_than_the_workspace_path():
    # 64 sequences x 64 query heads of D 128: the workspace path's split layout
    # (jl_decode_workspace_bytes) is larger than the fixed array, so the
    # no-allocation call runs with fewer splits.  Same results up to the order
    # of the final sum; both held to the oracle.
    B, L, Hq, Hkv, D, W, w0 = 64, 4096, 64, 8, 128, 1000, 300
    assert jl.jl_decode_workspace_bytes(B, L, Hq, Hkv, D) > FIXED_SCRATCH_BYTES
    dev = torch.device("cuda")
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    q, kc, vc = synthetic.decode_inputs(B, L, Hq, Hkv, D, seed=5, outlier_frac=0.01)
    q, kc, vc = q.to(dev), kc.to(dev), vc.to(dev)
    for _ in range(2):
        o_na, l_na = _noalloc_decode(q, kc, vc, L, w0, W, err)
        o_ref, l_ref = _workspace_decode(q, kc, vc, L, w0, W)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert (o_na.float() - o_ref.float()).abs().max().item() <= O_MAX_ABS
        assert (l_na - l_ref).abs().max().item() <= LSE_MAX_ABS
    _against_oracle(q[:4], kc[:4], vc[:4], o_na[:4], l_na[:4], L, w0, W, "noalloc, fewer splits")


def test_noalloc_decode_rejects_problems_beyond_its_fixed_scratch():
    # 4096 sequences x 64 query heads need 4096 * 64 * (4 * 128 + 8) bytes of
    # partials even with one split each: far more than the fixed array.
    dev = torch.device("cuda")
    q = torch.zeros(4096, 64, 128, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(4096, 64, 8, 128, dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    with pytest.raises(jl.JetLongError) as exc:
        jl.jl_bifocal_decode_noalloc(q, kc, kc, o, None, L=64, w0=8, w_pretrained=16, rope_base=1e6)
    assert exc.value.status == -4  # JL_ERR_WORKSPACE
