"""Multi-GPU layouts' kernels on one GPU, each "rank" run one after another (no
rank waits on another).  Sequence split: each rank is one key range of the
cache, and the partial results are merged by jl_decode_combine.  Head sharding:
each rank is one KV-head group with its query heads, as contiguous tensors of
its own.  The gathers themselves are covered over gloo in test_multigpu_cpu.py;
this file pins the kernels.
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


@pytest.mark.parametrize("world", [2, 4])
def test_head_shard_groups_equal_the_whole_problem(world):
    # Prefill and decode per KV-head group (the kernels see a smaller problem
    # with the same GQA ratio, G and band); concatenated over the groups they
    # equal one call on every head (prefill bit for bit: each head's result
    # does not depend on the others; decode within rounding, since the split
    # count follows the number of (sequence, KV head) pairs) and the oracle.
    B, L, Hq, Hkv, D, W, w0 = 1, 2000, 16, 4, 128, 600, 300
    q, k, v = synthetic.prefill_inputs(B, L, Hq, Hkv, D, seed=19, outlier_frac=0.01)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    kw = dict(w0=w0, w_pretrained=W, rope_base=1e6)
    o_all, l_all = multi_gpu.head_shard_prefill(qd, kd, vd, **kw)
    q1 = qd[:, L - 1].contiguous()
    od_all, ld_all = multi_gpu.head_shard_decode(q1, kd, vd, L=L, **kw)
    os_, ls_, ods, lds = [], [], [], []
    for rank in range(world):
        kb, kc_, qb, qc_ = multi_gpu.head_shard_slices(Hq, Hkv, rank, world)
        q_r = multi_gpu.take_heads(qd, qb, qc_)
        k_r, v_r = multi_gpu.take_heads(kd, kb, kc_), multi_gpu.take_heads(vd, kb, kc_)
        o_r, l_r = multi_gpu.head_shard_prefill(q_r, k_r, v_r, **kw)
        od_r, ld_r = multi_gpu.head_shard_decode(multi_gpu.take_heads(q1, qb, qc_, dim=1), k_r, v_r, L=L, **kw)
        os_.append(o_r)
        ls_.append(l_r)
        ods.append(od_r)
        lds.append(ld_r)
    torch.cuda.synchronize()
    o_sh, l_sh = torch.cat(os_, dim=2), torch.cat(ls_, dim=1)
    od_sh, ld_sh = torch.cat(ods, dim=1), torch.cat(lds, dim=1)
    assert torch.equal(o_sh, o_all) and torch.equal(l_sh, l_all)
    assert (od_sh.float() - od_all.float()).abs().max().item() <= 2e-2
    assert (ld_sh - ld_all).abs().max().item() <= 1e-3
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e6)
    rows = np.array([0, 299, 300, 301, 1023, 1024, 1999])
    ref = {}
    for h in (0, 5, 15):
        g = h // (Hq // Hkv)
        ref[h] = jo.attention_rows(q[0, rows, h].double().numpy(), rows, k[0, :, g].double().numpy(),
                                   v[0, :, g].double().numpy(), p)
        assert_close(o_sh[0, rows, h].float().cpu().numpy(), ref[h][0], l_sh[0, h, rows].cpu().numpy(), ref[h][1],
                     f"head shard h{h}")
    od_ref, ld_ref = jo.decode(q[:, L - 1].float().numpy(), k.float().numpy(), v.float().numpy(), p)
    assert_close(od_sh.float().cpu().numpy(), od_ref, ld_sh.cpu().numpy(), ld_ref, "head shard decode")
