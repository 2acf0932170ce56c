"""Sequence-split decode kernels on one GPU: each "rank" is one key range of
the cache, run one after another (no rank waits on another), then the partial
results are merged by jl_decode_combine.  The gather itself is covered over
gloo in test_multigpu_cpu.py; this file pins the kernels.
"""

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import multi_gpu, synthetic
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_context_extension_b200 import build
    build.build()


def _range(q, kc, vc, off, cnt, L, w0, W, base):
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    ks = kc[:, off:off + cnt].contiguous()   # this rank's shard, a buffer of its own
    vs = vc[:, off:off + cnt].contiguous()
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    ws = torch.zeros(jl.jl_decode_workspace_bytes(B, cnt, Hq, Hkv, D), dtype=torch.uint8, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    jl.jl_bifocal_decode_range(q, ks, vs, o, lse, key_offset=off, key_count=cnt, total_len=L, w0=w0,
                               w_pretrained=W, rope_base=base, workspace=ws, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return o, lse


@pytest.mark.parametrize("ranks", [2, 3, 8])
def test_key_ranges_combine_to_the_whole_decode(ranks):
    B, L, Hq, Hkv, D, W, w0, base = 2, 20000, 16, 2, 128, 7000, 500, 1e6   # G = 3
    q, kc, vc = synthetic.decode_inputs(B, L, Hq, Hkv, D, seed=51, outlier_frac=0.01)
    qd, kd, vd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=base)
    parts_o, parts_l = [], []
    for r in range(ranks):
        off, cnt = multi_gpu.shard_range(L, r, ranks)
        o_r, l_r = _range(qd, kd, vd, off, cnt, L, w0, W, base)
        o_ref, l_ref = jo.decode_key_range(q.double().numpy(), kc.double().numpy(), vc.double().numpy(), p, off,
                                           off + cnt)
        assert_close(o_r.float().cpu().numpy(), o_ref, l_r.cpu().numpy(), l_ref, f"range {r}/{ranks}")
        parts_o.append(o_r)
        parts_l.append(l_r)
    o = torch.empty_like(qd)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    jl.jl_decode_combine(torch.stack(parts_o).contiguous(), torch.stack(parts_l).contiguous(), o, lse)
    torch.cuda.synchronize()
    o_ref, l_ref = jo.decode(q.double().numpy(), kc.double().numpy(), vc.double().numpy(), p)
    assert_close(o.float().cpu().numpy(), o_ref, lse.cpu().numpy(), l_ref, f"combined over {ranks}")


def test_sequence_split_driver_single_rank_equals_decode():
    B, L, Hq, Hkv, D, W, w0, base = 1, 9000, 8, 1, 64, 4000, 300, 1e6
    q, kc, vc = synthetic.decode_inputs(B, L, Hq, Hkv, D, seed=52)
    qd, kd, vd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    o, lse = multi_gpu.sequence_split_decode(qd, kd, vd, key_offset=0, key_count=L, total_len=L, w0=w0,
                                             w_pretrained=W, rope_base=base)
    torch.cuda.synchronize()
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=base)
    o_ref, l_ref = jo.decode(q.double().numpy(), kc.double().numpy(), vc.double().numpy(), p)
    assert_close(o.float().cpu().numpy(), o_ref, lse.cpu().numpy(), l_ref, "driver, one rank")
