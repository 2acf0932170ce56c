"""Seeded randomized parity sweep (GPU, through the C ABI, against the fp64 oracle).

The shapes, band widths, group sizes, query-shift modes and precisions come from
a fixed seed, so the sweep is the same on every run: ragged lengths (1 .. 640),
odd and even GQA ratios (one or two heads per CTA), both head dims, w0 at tile
edges, at L - 1, L and beyond, and G from 1 to 8.  Every case is small enough
for the dense oracle, so whole outputs are compared.
"""

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic
from tests.gpu_helpers import MODES, assert_close, run_decode, run_prefill

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_context_extension_b200 import build
    build.build()


def _draw(rng, L):
    """Head layout, band width, w_pretrained (for a target G) and mode for length L."""
    D = int(rng.choice([64, 128]))
    Hkv = int(rng.choice([1, 2, 3]))
    r = int(rng.choice([1, 2, 3, 4]))
    G = int(rng.integers(1, 9))
    W = max(1, -(-L // G))
    w0 = int(rng.choice([0, 1, 127, 128, 129, max(0, L - 1), L, L + 5, int(rng.integers(0, L + 1))]))
    mode = str(rng.choice([jo.MODE_SELF_EXTEND, jo.MODE_NONE]))
    return D, Hkv * r, Hkv, W, w0, mode


def _prefill_cases(n=40, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        L = int(rng.integers(1, 641))
        D, Hq, Hkv, W, w0, mode = _draw(rng, L)
        B = int(rng.integers(1, 3))
        u = rng.random()
        prec = "inkernel" if u < 0.2 else ("fp16" if u < 0.35 else "default")
        outl = 0.0 if prec == "fp16" else float(rng.choice([0.0, 0.01]))
        cases.append((B, L, Hq, Hkv, D, W, w0, mode, prec, outl))
    return cases


def _decode_cases(n=40, seed=7):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        Lmax = int(rng.integers(1, 5001))
        L = int(rng.integers(1, Lmax + 1))
        D, Hq, Hkv, W, w0, mode = _draw(rng, L)
        B = int(rng.integers(1, 4))
        cases.append((B, Lmax, L, Hq, Hkv, D, W, w0, mode))
    return cases


@pytest.mark.parametrize("B,L,Hq,Hkv,D,W,w0,mode,prec,outl", _prefill_cases())
def test_prefill_random_shapes(B, L, Hq, Hkv, D, W, w0, mode, prec, outl):
    q, k, v = synthetic.prefill_inputs(B, L, Hq, Hkv, D, seed=L * 7 + Hq, outlier_frac=outl)
    o, lse, err = run_prefill(q, k, v, w0=w0, W=W, base=10000.0, mode=mode, prec=prec)
    assert err == 0
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=10000.0, mode=mode)
    o_ref, lse_ref = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    assert_close(o.numpy(), o_ref, lse.numpy(), lse_ref,
                 f"B{B} L{L} {Hq}/{Hkv} d{D} W{W} w0{w0} {mode} {prec} outliers {outl}")


@pytest.mark.parametrize("B,Lmax,L,Hq,Hkv,D,W,w0,mode", _decode_cases())
def test_decode_random_shapes(B, Lmax, L, Hq, Hkv, D, W, w0, mode):
    q, kc, vc = synthetic.decode_inputs(B, Lmax, Hq, Hkv, D, seed=L + Lmax, length=L)
    o, lse, err = run_decode(q, kc, vc, L=L, w0=w0, W=W, base=10000.0, mode=mode)
    assert err == 0
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=10000.0, mode=mode)
    o_ref, lse_ref = jo.decode(q.float().numpy(), kc.float().numpy(), vc.float().numpy(), p)
    assert_close(o.numpy(), o_ref, lse.numpy(), lse_ref, f"B{B} Lmax{Lmax} L{L} {Hq}/{Hkv} d{D} W{W} w0{w0} {mode}")


def _chunk_cases(n=16, seed=99):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        total = int(rng.integers(2, 641))
        P = int(rng.integers(0, total))
        D, Hq, Hkv, W, w0, mode = _draw(rng, total)
        cases.append((P, total - P, Hq, Hkv, D, W, w0, mode))
    return cases


@pytest.mark.parametrize("P,C,Hq,Hkv,D,W,w0,mode", _chunk_cases())
def test_chunked_prefill_random_shapes(P, C, Hq, Hkv, D, W, w0, mode):
    # a chunk of C queries at positions P .. P + C - 1 against a cache of P + C keys
    q_full, k, v = synthetic.prefill_inputs(1, P + C, Hq, Hkv, D, seed=P + 3 * C)
    q = q_full[:, P:P + C].contiguous().to(DEV)
    kd, vd = k.to(DEV), v.to(DEV)
    o = torch.empty_like(q)
    lse = torch.empty(1, Hq, C, dtype=torch.float32, device=DEV)
    ws = torch.empty(jl.jl_prefill_chunk_workspace_bytes(1, P, C, Hq, Hkv, D), dtype=torch.uint8, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    jl.jl_bifocal_prefill_chunk(q, kd, vd, o, lse, q_offset=P, w0=w0, w_pretrained=W, rope_base=10000.0,
                                mode=MODES[mode], workspace=ws, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    p = jo.BifocalParams(L=P + C, w0=w0, w_pretrained=W, base=10000.0, mode=mode)
    o_ref, lse_ref = jo.prefill_dense(q_full.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    assert_close(o.float().cpu().numpy(), o_ref[:, P:], lse.cpu().numpy(), lse_ref[:, :, P:],
                 f"chunk P{P} C{C} {Hq}/{Hkv} d{D} W{W} w0{w0} {mode}")
