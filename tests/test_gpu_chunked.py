"""Chunked prefill against an existing cache (GPU, through the C ABI, against
the fp64 oracle).

A chunk's queries sit at positions P .. P + C - 1 and attend to cache keys
0 .. P + C - 1, with G from the total length P + C (the current length, Jet-Long
review "Method").  Rows of a chunk are exact rows of the whole-sequence
prefill at that total length.
"""

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic
from tests.gpu_helpers import PRECISIONS, prefill_workspace, MODES, assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_context_extension_b200 import build
    build.build()


def _chunk(q, kc, vc, P, w0, W, base, mode=jo.MODE_SELF_EXTEND, prec="default"):
    B, C, Hq, D = q.shape
    Hkv = kc.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, C, dtype=torch.float32, device=DEV)
    ws = prefill_workspace(prec, jl.jl_prefill_chunk_workspace_bytes(B, P, C, Hq, Hkv, D), DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    m = MODES[mode] | PRECISIONS[prec]
    jl.jl_bifocal_prefill_chunk(q, kc, vc, o, lse, q_offset=P, w0=w0, w_pretrained=W, rope_base=base, mode=m,
                                workspace=ws, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return o.float().cpu(), lse.cpu()


def _oracle_chunk(q_full, k, v, P, C, w0, W, base, mode=jo.MODE_SELF_EXTEND):
    p = jo.BifocalParams(L=P + C, w0=w0, w_pretrained=W, base=base, mode=mode)
    res = jo.prefill(q_full[:, :P + C].float().numpy(), k[:, :P + C].float().numpy(), v[:, :P + C].float().numpy(),
                     p, rows=np.arange(P, P + C))
    B, _, Hq, D = q_full.shape
    o = np.zeros((B, C, Hq, D))
    lse = np.zeros((B, Hq, C))
    for (b, h), (_, ob, lb) in res.items():
        o[b, :, h] = ob
        lse[b, h] = lb
    return o, lse


@pytest.mark.parametrize("P,C,w0,W,mode,prec,outl", [
    (0, 1500, 200, 400, jo.MODE_SELF_EXTEND, "default", 0.01),   # whole sequence from a cache
    (700, 800, 200, 400, jo.MODE_SELF_EXTEND, "default", 0.01),  # offset not a multiple of the 128-row tile
    (1300, 200, 200, 400, jo.MODE_NONE, "default", 0.0),
    (1111, 389, 0, 400, jo.MODE_SELF_EXTEND, "default", 0.01),   # w0 = 0: every pair remote
    (5, 50, 16, 20, jo.MODE_SELF_EXTEND, "default", 0.0),        # small chunk, stale rows after it in the cache
    (900, 600, 200, 1600, jo.MODE_SELF_EXTEND, "default", 0.0),  # G = 1 at the total length: plain causal RoPE
    (700, 800, 200, 400, jo.MODE_SELF_EXTEND, "inkernel", 0.01),  # key tiles corrected in the kernel
    (700, 800, 200, 400, jo.MODE_SELF_EXTEND, "fp16", 0.0),      # single fp16 product
])
def test_chunk_matches_oracle(P, C, w0, W, mode, prec, outl):
    Lmax = P + C + 77
    q_full, k, v = synthetic.prefill_inputs(1, Lmax, 8, 2, 128, seed=P + C, outlier_frac=outl)
    qc = q_full[:, P:P + C].contiguous()
    o, lse = _chunk(qc.to(DEV), k.to(DEV), v.to(DEV), P, w0, W, 1e6, mode, prec)
    o_ref, lse_ref = _oracle_chunk(q_full, k, v, P, C, w0, W, 1e6, mode)
    assert_close(o.numpy(), o_ref, lse.numpy(), lse_ref, f"chunk P{P} C{C}")


def test_final_chunk_equals_whole_prefill_rows():
    # Same total length, hence same G: the last chunk reproduces the rows of
    # the one-shot prefill, and cache rows past the chunk do not matter.
    L, P, W, w0 = 2000, 1234, 512, 300
    q, k, v = synthetic.prefill_inputs(1, L, 8, 2, 128, seed=31)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o_full = torch.empty_like(qd)
    lse_full = torch.empty(1, 8, L, dtype=torch.float32, device=DEV)
    ws = torch.empty(jl.jl_prefill_workspace_bytes(1, L, 8, 2, 128), dtype=torch.uint8, device=DEV)
    jl.jl_bifocal_prefill(qd, kd, vd, o_full, lse_full, w0=w0, w_pretrained=W, rope_base=1e6, workspace=ws)
    kbig = torch.cat([kd, torch.full((1, 300, 2, 128), 7.0, dtype=torch.bfloat16, device=DEV)], dim=1)
    vbig = torch.cat([vd, torch.full((1, 300, 2, 128), -7.0, dtype=torch.bfloat16, device=DEV)], dim=1)
    o_c, lse_c = _chunk(qd[:, P:].contiguous(), kbig, vbig, P, w0, W, 1e6)
    torch.cuda.synchronize()
    assert (o_c - o_full[:, P:].float().cpu()).abs().max() <= 2e-2
    assert (lse_c - lse_full[:, :, P:].cpu()).abs().max() <= 1e-3
