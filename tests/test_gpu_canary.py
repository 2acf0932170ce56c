"""Out-of-bounds writes, checked without a sanitizer.

Every output and scratch buffer is carved out of a larger allocation whose
margins (256 bytes on each side) hold a known byte pattern; after the call the
margins must be untouched, the inputs (and the KV cache) unchanged, and the
outputs equal, bit for bit, to those of the same call on plain buffers.
Shapes are ragged (lengths off the tile sizes, several batches) so that every
edge tile and every tail mask is exercised.
"""

import numpy as np
import pytest
import torch

from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic
from tests.gpu_helpers import PRECISIONS

pytestmark = pytest.mark.gpu

PAD = 256
FILL = 0x5A
DEV = torch.device("cuda")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_context_extension_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _padded(shape, dtype):
    nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((PAD + nbytes + PAD,), FILL, dtype=torch.uint8, device=DEV)
    return raw, raw[PAD:PAD + nbytes].view(dtype).view(*shape)


def _margins_intact(raw, what):
    assert bool((raw[:PAD] == FILL).all()), f"{what}: write before the buffer"
    assert bool((raw[-PAD:] == FILL).all()), f"{what}: write past the buffer"


@pytest.mark.parametrize("prec", ["default", "inkernel", "fp16"])
def test_prefill_writes_only_its_outputs(prec):
    # (the workspace, where the mode takes one, is checked like the outputs)
    B, L, Hq, Hkv, D, W, w0 = 2, 700, 4, 2, 128, 200, 150
    q, k, v = synthetic.prefill_inputs(B, L, Hq, Hkv, D, seed=31, outlier_frac=0.01)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    q0, k0, v0 = qd.clone(), kd.clone(), vd.clone()
    mode = jl.JL_QSHIFT_SELF_EXTEND | PRECISIONS[prec]
    ws_bytes = 0 if prec == "inkernel" else jl.jl_prefill_workspace_bytes(B, L, Hq, Hkv, D)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)

    o_raw, o = _padded((B, L, Hq, D), torch.bfloat16)
    l_raw, lse = _padded((B, Hq, L), torch.float32)
    w_raw, ws = _padded((ws_bytes,), torch.uint8) if ws_bytes else (None, None)
    jl.jl_bifocal_prefill(qd, kd, vd, o, lse, w0=w0, w_pretrained=W, rope_base=1e6, mode=mode, workspace=ws,
                          dev_error=err)
    torch.cuda.synchronize()
    for raw, what in ((o_raw, "O"), (l_raw, "LSE"), (w_raw, "workspace")):
        if raw is not None:
            _margins_intact(raw, what)
    assert torch.equal(qd, q0) and torch.equal(kd, k0) and torch.equal(vd, v0), "inputs were written"

    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    ws2 = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV) if ws_bytes else None
    jl.jl_bifocal_prefill(qd, kd, vd, o2, lse2, w0=w0, w_pretrained=W, rope_base=1e6, mode=mode, workspace=ws2,
                          dev_error=err)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert int(err.item()) == 0


def test_decode_writes_only_its_outputs():
    B, Lmax, L, Hq, Hkv, D, W, w0 = 3, 2200, 2000, 8, 2, 128, 600, 300
    q, kc, vc = synthetic.decode_inputs(B, Lmax, Hq, Hkv, D, seed=32, outlier_frac=0.01)
    qd, kd, vd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    q0, k0, v0 = qd.clone(), kd.clone(), vd.clone()
    ws_bytes = jl.jl_decode_workspace_bytes(B, L, Hq, Hkv, D)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)

    o_raw, o = _padded((B, Hq, D), torch.bfloat16)
    l_raw, lse = _padded((B, Hq), torch.float32)
    w_raw = torch.full((PAD + ws_bytes + PAD,), FILL, dtype=torch.uint8, device=DEV)
    ws = w_raw[PAD:PAD + ws_bytes]
    ws.zero_()  # ticket counters start at zero
    for _ in range(2):  # the second call reuses the counters the first left at zero
        jl.jl_bifocal_decode(qd, kd, vd, o, lse, L=L, w0=w0, w_pretrained=W, rope_base=1e6, workspace=ws,
                             dev_error=err)
    torch.cuda.synchronize()
    for raw, what in ((o_raw, "O"), (l_raw, "LSE"), (w_raw, "workspace")):
        _margins_intact(raw, what)
    assert torch.equal(qd, q0) and torch.equal(kd, k0) and torch.equal(vd, v0), "inputs or cache were written"

    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    ws2 = torch.zeros(ws_bytes, dtype=torch.uint8, device=DEV)
    jl.jl_bifocal_decode(qd, kd, vd, o2, lse2, L=L, w0=w0, w_pretrained=W, rope_base=1e6, workspace=ws2,
                         dev_error=err)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert int(err.item()) == 0


def test_chunked_prefill_writes_only_its_outputs():
    B, Lmax, P, C, Hq, Hkv, D, W, w0 = 2, 1100, 333, 500, 4, 2, 128, 250, 120
    q_all, kc, vc = synthetic.prefill_inputs(B, Lmax, Hq, Hkv, D, seed=33)
    qd = q_all[:, P:P + C].contiguous().to(DEV)
    kd, vd = kc.to(DEV), vc.to(DEV)
    k0, v0 = kd.clone(), vd.clone()
    ws_bytes = jl.jl_prefill_chunk_workspace_bytes(B, P, C, Hq, Hkv, D)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    o_raw, o = _padded((B, C, Hq, D), torch.bfloat16)
    l_raw, lse = _padded((B, Hq, C), torch.float32)
    w_raw, ws = _padded((ws_bytes,), torch.uint8)
    jl.jl_bifocal_prefill_chunk(qd, kd, vd, o, lse, q_offset=P, w0=w0, w_pretrained=W, rope_base=1e6,
                                workspace=ws, dev_error=err)
    torch.cuda.synchronize()
    for raw, what in ((o_raw, "O"), (l_raw, "LSE"), (w_raw, "workspace")):
        _margins_intact(raw, what)
    assert torch.equal(kd, k0) and torch.equal(vd, v0), "cache was written"
    # the key tiles corrected in the kernel (no workspace) on the same chunk:
    # same outputs within rounding, margins intact
    o3_raw, o3 = _padded((B, C, Hq, D), torch.bfloat16)
    l3_raw, lse3 = _padded((B, Hq, C), torch.float32)
    jl.jl_bifocal_prefill_chunk(qd, kd, vd, o3, lse3, q_offset=P, w0=w0, w_pretrained=W, rope_base=1e6,
                                mode=jl.JL_QSHIFT_SELF_EXTEND | jl.JL_PREFILL_KEYS_IN_KERNEL, dev_error=err)
    torch.cuda.synchronize()
    _margins_intact(o3_raw, "O (default)")
    _margins_intact(l3_raw, "LSE (default)")
    assert (o3.float() - o.float()).abs().max().item() <= 1.6e-2
    assert torch.equal(kd, k0) and torch.equal(vd, v0), "cache was written"
    assert int(err.item()) == 0
