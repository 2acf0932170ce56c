"""The C-ABI entry points inside CUDA graphs.

A serving loop captures a decode step (and often a prefill) once and replays
it, so the host cost of argument checks, tensor-map encoding and the launch is
paid once.  These tests capture the calls with torch's graph API on the
caller's stream and check that every replay gives, bit for bit, what an eager
call on the same inputs gives: also after the inputs are rewritten between
replays (the graph must read the buffers, not anything cached at capture) and
for the decode scratch, whose ticket counters the last CTA resets for the next
launch.  One eager result per entry point is also held to the fp64 oracle.
"""

import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_context_extension_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _capture(fn, n_calls):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm-up on the capture stream (lazy attribute set-up, first-launch work)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n_calls):
            fn()
    return g


def test_decode_graph_replay_matches_eager():
    B, L, Hq, Hkv, D, W, w0 = 2, 5000, 8, 2, 128, 1500, 300  # G 4, ragged tiles
    dev = torch.device("cuda")
    q, kc, vc = synthetic.decode_inputs(B, L, Hq, Hkv, D, seed=11, outlier_frac=0.01)
    q2, _, _ = synthetic.decode_inputs(B, L, Hq, Hkv, D, seed=12)
    qd, kd, vd = q.to(dev), kc.to(dev), vc.to(dev)
    o = torch.empty_like(qd)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = torch.zeros(jl.jl_decode_workspace_bytes(B, L, Hq, Hkv, D), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        jl.jl_bifocal_decode(qd, kd, vd, o, lse, L=L, w0=w0, w_pretrained=W, rope_base=1e6, workspace=ws,
                             dev_error=err)

    call()
    torch.cuda.synchronize()
    o_eager, lse_eager = o.clone(), lse.clone()
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e6)
    o_ref, lse_ref = jo.decode(q.double().numpy(), kc.double().numpy(), vc.double().numpy(), p)
    assert_close(o_eager.float().cpu().numpy(), o_ref, lse_eager.cpu().numpy(), lse_ref, "decode eager")

    g = _capture(call, 2)  # two launches in one graph: the counters must be reset in between
    for _ in range(3):
        o.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_eager) and torch.equal(lse, lse_eager)

    # new query values in the captured buffer: the replay must see them
    qd.copy_(q2.to(dev))
    g.replay()
    torch.cuda.synchronize()
    o_g, lse_g = o.clone(), lse.clone()
    call()
    torch.cuda.synchronize()
    assert torch.equal(o_g, o) and torch.equal(lse_g, lse)
    assert not torch.equal(o_g, o_eager)
    assert int(err.item()) == 0


def test_prefill_graph_replay_matches_eager():
    B, L, Hq, Hkv, D, W, w0 = 1, 1000, 4, 2, 128, 300, 200  # G 4, ragged tiles, straddling band
    dev = torch.device("cuda")
    q, k, v = synthetic.prefill_inputs(B, L, Hq, Hkv, D, seed=21)
    q2, _, _ = synthetic.prefill_inputs(B, L, Hq, Hkv, D, seed=22)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty_like(qd)
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)
    ws = torch.empty(jl.jl_prefill_workspace_bytes(B, L, Hq, Hkv, D), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        jl.jl_bifocal_prefill(qd, kd, vd, o, lse, w0=w0, w_pretrained=W, rope_base=1e6, workspace=ws,
                              dev_error=err)

    call()
    torch.cuda.synchronize()
    o_eager, lse_eager = o.clone(), lse.clone()
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=1e6)
    o_ref, lse_ref = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    assert_close(o_eager.float().cpu().numpy(), o_ref, lse_eager.cpu().numpy(), lse_ref, "prefill eager")

    g = _capture(call, 1)
    for _ in range(3):
        o.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_eager) and torch.equal(lse, lse_eager)

    qd.copy_(q2.to(dev))
    g.replay()
    torch.cuda.synchronize()
    o_g, lse_g = o.clone(), lse.clone()
    call()
    torch.cuda.synchronize()
    assert torch.equal(o_g, o) and torch.equal(lse_g, lse)
    assert not torch.equal(o_g, o_eager)
    assert int(err.item()) == 0
