"""Multi-GPU layouts across ranks, on CPU: world size 2 over gloo.

Sequence-split decode: each rank owns one key range of the cache.  The rank's
partial result comes from the fp64 oracle restricted to that range (the GPU
kernel stands in for it on the GPU side), the gather runs over gloo through
multi_gpu.sequence_split_decode, and a plain log-sum-exp combine must
reproduce the oracle's decode over the whole cache.

Head sharding: each rank owns a group of KV heads and their query heads; its
result (the oracle on the rank's heads alone) is gathered over gloo by
multi_gpu.head_shard_prefill / head_shard_decode and must equal the oracle on
every head.  Also pins the range partition and the head sharding.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _lse_combine(o_parts, lse_parts):
    m = lse_parts.max(dim=0).values
    w = torch.exp(lse_parts - m)
    den = w.sum(dim=0)
    return (w.unsqueeze(-1) * o_parts).sum(dim=0) / den.unsqueeze(-1), m + torch.log(den)


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    from oracle import jetlong_oracle as jo
    from rope_context_extension_b200 import multi_gpu, synthetic
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    L, W, w0 = 1500, 400, 200
    q, kc, vc = synthetic.decode_inputs(2, L, 8, 2, 64, seed=41, outlier_frac=0.01)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e4)
    off, cnt = multi_gpu.shard_range(L, rank, world)

    def partial(qq, ks, vs, key_offset, key_count, total_len, kw):
        o, lse = jo.decode_key_range(qq.double().numpy(), kc.double().numpy(), vc.double().numpy(), p,
                                     key_offset, key_offset + key_count)
        return torch.from_numpy(o), torch.from_numpy(lse)

    o, lse = multi_gpu.sequence_split_decode(q, kc[:, off:off + cnt], vc[:, off:off + cnt], key_offset=off,
                                             key_count=cnt, total_len=L, partial_fn=partial,
                                             combine_fn=_lse_combine)
    o_ref, lse_ref = jo.decode(q.double().numpy(), kc.double().numpy(), vc.double().numpy(), p)
    out.put((rank, float(np.abs(o.numpy() - o_ref).max()), float(np.abs(lse.numpy() - lse_ref).max())))
    dist.barrier()
    dist.destroy_process_group()


def test_sequence_split_decode_world2_matches_whole_cache():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, e_o, e_l in res:
        assert e_o < 1e-12 and e_l < 1e-12, (rank, e_o, e_l)


def _head_worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    from oracle import jetlong_oracle as jo
    from rope_context_extension_b200 import multi_gpu, synthetic
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    B, L, Hq, Hkv, D, W, w0 = 2, 300, 8, 4, 32, 80, 40
    q, k, v = synthetic.prefill_inputs(B, L, Hq, Hkv, D, seed=43, outlier_frac=0.01)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e4)
    kb, kc_, qb, qc_ = multi_gpu.head_shard_slices(Hq, Hkv, rank, world)
    q_r, k_r, v_r = (multi_gpu.take_heads(t, b_, c_) for t, b_, c_ in ((q, qb, qc_), (k, kb, kc_), (v, kb, kc_)))

    def prefill(qq, kk, vv, kw):  # the oracle on this rank's heads alone
        o, lse = jo.prefill_dense(qq.double().numpy(), kk.double().numpy(), vv.double().numpy(), p)
        return torch.from_numpy(o), torch.from_numpy(lse)

    o, lse = multi_gpu.head_shard_prefill(q_r, k_r, v_r, gather=True, prefill_fn=prefill)
    o_ref, lse_ref = jo.prefill_dense(q.double().numpy(), k.double().numpy(), v.double().numpy(), p)
    e_pre = (float(np.abs(o.numpy() - o_ref).max()), float(np.abs(lse.numpy() - lse_ref).max()))
    # decode of the last token against the same keys
    qd = q[:, L - 1].contiguous()
    qd_r = multi_gpu.take_heads(qd, qb, qc_, dim=1)

    def decode(qq, kk, vv, kw):
        o_, l_ = jo.decode(qq.double().numpy(), kk.double().numpy(), vv.double().numpy(), p)
        return torch.from_numpy(o_), torch.from_numpy(l_)

    od, ld = multi_gpu.head_shard_decode(qd_r, k_r, v_r, gather=True, decode_fn=decode, L=L)
    od_ref, ld_ref = jo.decode(qd.double().numpy(), k.double().numpy(), v.double().numpy(), p)
    e_dec = (float(np.abs(od.numpy() - od_ref).max()), float(np.abs(ld.numpy() - ld_ref).max()))
    out.put((rank, e_pre, e_dec, tuple(o.shape), tuple(lse.shape), tuple(od.shape)))
    dist.barrier()
    dist.destroy_process_group()


def test_head_shard_world2_gathers_every_head():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, e_pre, e_dec, so, sl, sd in res:
        assert so == (2, 300, 8, 32) and sl == (2, 8, 300) and sd == (2, 8, 32)
        # each head's result is computed by the same arithmetic on either side
        assert max(e_pre) == 0.0 and max(e_dec) == 0.0, (rank, e_pre, e_dec)


def test_head_shard_slices():
    from rope_context_extension_b200 import multi_gpu
    assert [multi_gpu.head_shard_slices(32, 8, r, 4) for r in range(4)] == \
        [(0, 2, 0, 8), (2, 2, 8, 8), (4, 2, 16, 8), (6, 2, 24, 8)]
    with pytest.raises(ValueError):
        multi_gpu.head_shard_slices(30, 8, 0, 2)


def test_shard_range_and_head_shard():
    from rope_context_extension_b200 import multi_gpu
    for total in (1, 7, 131072, 100003):
        for world in (1, 2, 3, 8):
            parts = [multi_gpu.shard_range(total, r, world) for r in range(world)]
            assert parts[0][0] == 0
            for (b0, c0), (b1, _) in zip(parts, parts[1:]):
                assert b0 + c0 == b1
            assert sum(c for _, c in parts) == total
    assert [multi_gpu.head_shard(8, r, 4) for r in range(4)] == [(0, 2), (2, 2), (4, 2), (6, 2)]
    with pytest.raises(ValueError):
        multi_gpu.head_shard(8, 0, 3)


def test_oracle_key_ranges_combine_to_the_whole():
    # the decomposition itself, in one process: disjoint ranges merged by LSE = the whole decode
    from oracle import jetlong_oracle as jo
    from rope_context_extension_b200 import synthetic
    L = 900
    q, kc, vc = synthetic.decode_inputs(1, L, 4, 1, 32, seed=42)
    p = jo.BifocalParams(L=L, w0=100, w_pretrained=200, base=1e4)
    cuts = [0, 10, 450, 899, 900]
    parts = [jo.decode_key_range(q.double().numpy(), kc.double().numpy(), vc.double().numpy(), p, a, b)
             for a, b in zip(cuts, cuts[1:])]
    o, lse = _lse_combine(torch.stack([torch.from_numpy(x[0]) for x in parts]),
                          torch.stack([torch.from_numpy(x[1]) for x in parts]))
    o_ref, lse_ref = jo.decode(q.double().numpy(), kc.double().numpy(), vc.double().numpy(), p)
    np.testing.assert_allclose(o.numpy(), o_ref, atol=1e-12)
    np.testing.assert_allclose(lse.numpy(), lse_ref, atol=1e-12)
