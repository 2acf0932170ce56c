"""Varlen decode, base-RoPE cache append, and streaming generation across a
group-size boundary (GPU, through the C ABI, against the fp64 oracle).

The Jet-Long pages claim that keeping base keys in the cache and correcting
them on the fly lets generation stream across length boundaries (where G
changes) without rewriting the cache (gist.science summary, "§2 On-the-Fly
Correctie Rotatie").  These tests run that loop: each step rotates and appends
the new token, then decodes every sequence of the batch at its own length.
"""

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_context_extension_b200 import build
    build.build()


def _oracle_varlen(q, kc, vc, lens, w0, W, base, mode=jo.MODE_SELF_EXTEND):
    outs, lses = [], []
    for b, L in enumerate(lens):
        p = jo.BifocalParams(L=int(L), w0=w0, w_pretrained=W, base=base, mode=mode)
        o, lse = jo.decode(q[b:b + 1].double().numpy(), kc[b:b + 1].double().numpy(), vc[b:b + 1].double().numpy(),
                           p)
        outs.append(o[0])
        lses.append(lse[0])
    return np.stack(outs), np.stack(lses)


def _varlen(q, kc, vc, lens, w0, W, base, mode=jl.JL_QSHIFT_SELF_EXTEND):
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    ws = torch.zeros(jl.jl_decode_workspace_bytes(B, max(lens), Hq, Hkv, D), dtype=torch.uint8, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    jl.jl_bifocal_decode_varlen(q, kc, vc, o, lse, sl, max_len=max(lens), w0=w0, w_pretrained=W, rope_base=base,
                                mode=mode, workspace=ws, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return o.float().cpu(), lse.cpu()


@pytest.mark.parametrize("mode", [jo.MODE_SELF_EXTEND, jo.MODE_NONE])
def test_varlen_batch_spans_group_sizes(mode):
    # one batch, four sequences with G = 1, 2, 3, 4 (w_pretrained 1000)
    lens = [700, 1999, 2001, 4000]
    W, w0 = 1000, 150
    q, kc, vc = synthetic.decode_inputs(4, 4096, 8, 2, 128, seed=21, outlier_frac=0.01)
    o, lse = _varlen(q.to(DEV), kc.to(DEV), vc.to(DEV), lens, w0, W, 1e6,
                     jl.JL_QSHIFT_SELF_EXTEND if mode == jo.MODE_SELF_EXTEND else jl.JL_QSHIFT_NONE)
    o_ref, lse_ref = _oracle_varlen(q, kc, vc, lens, w0, W, 1e6, mode)
    assert_close(o.numpy(), o_ref, lse.numpy(), lse_ref, "varlen")


def test_varlen_matches_uniform_decode_when_lengths_are_equal():
    q, kc, vc = synthetic.decode_inputs(3, 3000, 8, 2, 64, seed=22)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    o1, l1 = _varlen(q, kc, vc, [2500, 2500, 2500], 200, 1024, 1e4)
    o2 = torch.empty_like(q)
    l2 = torch.empty(3, 8, dtype=torch.float32, device=DEV)
    ws = torch.zeros(jl.jl_decode_workspace_bytes(3, 2500, 8, 2, 64), dtype=torch.uint8, device=DEV)
    jl.jl_bifocal_decode(q, kc, vc, o2, l2, L=2500, w0=200, w_pretrained=1024, rope_base=1e4, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2.float().cpu()) and torch.equal(l1, l2.cpu())


def test_rope_append_rotates_and_writes_one_row():
    B, Hq, Hkv, D, Lmax, base = 3, 8, 2, 128, 5000, 1e6
    g = torch.Generator("cpu").manual_seed(23)
    q_raw = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    k_raw = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)
    v_new = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Lmax, Hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Lmax, Hkv, D, generator=g).to(torch.bfloat16)
    pos = [0, 1234, 4999]
    kd, vd = kc.to(DEV), vc.to(DEV)
    q_out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=DEV)
    jl.jl_rope_append(q_raw.to(DEV), k_raw.to(DEV), v_new.to(DEV), torch.tensor(pos, dtype=torch.int32, device=DEV),
                      q_out, kd, vd, rope_base=base)
    torch.cuda.synchronize()
    kd, vd, q_out = kd.cpu(), vd.cpu(), q_out.cpu()
    for b, p in enumerate(pos):
        want_q = jo.rope_rotate(q_raw[b].double().numpy(), p, base)
        want_k = jo.rope_rotate(k_raw[b].double().numpy(), p, base)
        # bf16 round-to-nearest of the fp64 rotation: within half an ulp (2^-9 relative) plus fp32 slack
        tol_q = np.abs(want_q) * 2.0 ** -8 + 1e-6
        tol_k = np.abs(want_k) * 2.0 ** -8 + 1e-6
        assert np.all(np.abs(q_out[b].double().numpy() - want_q) <= tol_q)
        assert np.all(np.abs(kd[b, p].double().numpy() - want_k) <= tol_k)
        assert torch.equal(vd[b, p], v_new[b])
        # every other row untouched
        mask = torch.ones(Lmax, dtype=torch.bool)
        mask[p] = False
        assert torch.equal(kd[b][mask], kc[b][mask]) and torch.equal(vd[b][mask], vc[b][mask])


def test_streaming_generation_across_the_group_boundary():
    # Sequences start just below w_pretrained and generate past it, so G goes
    # from 1 to 2 mid-stream (and from 2 to 3 for the longest one); the cache
    # rows already written are never rewritten and every step matches the
    # oracle at that step's length.
    B, Hq, Hkv, D, W, w0, base = 3, 8, 2, 128, 256, 64, 1e6
    start = [250, 240, 505]
    steps = 12
    Lmax = max(start) + steps
    g = torch.Generator("cpu").manual_seed(24)
    kc = torch.zeros(B, Lmax, Hkv, D, dtype=torch.bfloat16)
    vc = torch.zeros(B, Lmax, Hkv, D, dtype=torch.bfloat16)
    # the prompt: raw keys rotated at their base positions (oracle rotation, rounded to bf16)
    for b, n in enumerate(start):
        kr = torch.randn(n, Hkv, D, generator=g).double().numpy()
        kc[b, :n] = torch.from_numpy(jo.rope_rotate(kr, np.arange(n)[:, None], base)).to(torch.bfloat16)
        vc[b, :n] = torch.randn(n, Hkv, D, generator=g).to(torch.bfloat16)
    kd, vd = kc.to(DEV), vc.to(DEV)
    ws = torch.zeros(jl.jl_decode_workspace_bytes(B, Lmax, Hq, Hkv, D), dtype=torch.uint8, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    seen_g = set()
    for t in range(steps):
        pos = [n + t for n in start]
        q_raw = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
        k_raw = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)
        v_new = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)
        before = kd.clone()
        q_rot = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=DEV)
        pd = torch.tensor(pos, dtype=torch.int32, device=DEV)
        jl.jl_rope_append(q_raw.to(DEV), k_raw.to(DEV), v_new.to(DEV), pd, q_rot, kd, vd, rope_base=base,
                          dev_error=err)
        lens = [p + 1 for p in pos]
        o = torch.empty_like(q_rot)
        lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
        jl.jl_bifocal_decode_varlen(q_rot, kd, vd, o, lse, pd + 1, max_len=max(lens), w0=w0, w_pretrained=W,
                                    rope_base=base, workspace=ws, dev_error=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        # only the appended rows changed
        changed = (kd != before).any(dim=-1).any(dim=-1).cpu()
        for b in range(B):
            rows = torch.nonzero(changed[b]).flatten().tolist()
            assert set(rows) <= {pos[b]}
        seen_g |= {jo.group_size(L, W) for L in lens}
        o_ref, lse_ref = _oracle_varlen(q_rot.cpu(), kd.cpu(), vd.cpu(), lens, w0, W, base)
        assert_close(o.float().cpu().numpy(), o_ref, lse.cpu().numpy(), lse_ref, f"stream step {t}")
    assert {1, 2, 3} <= seen_g
