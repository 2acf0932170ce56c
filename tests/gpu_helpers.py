"""Shared helpers for the GPU parity tests: run the library through the C-ABI
binding and compare with the fp64 oracle on the same seeded inputs."""

from __future__ import annotations

import numpy as np
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl
from rope_context_extension_b200 import synthetic

# Tolerances against the fp64 oracle (bf16 outputs, fp32 LSE), for every path
# and every input, outliers included.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3

MODES = {jo.MODE_NONE: jl.JL_QSHIFT_NONE, jo.MODE_SELF_EXTEND: jl.JL_QSHIFT_SELF_EXTEND}
# Prefill variants: the default (hi + lo remote operands; query rows corrected in
# the attention kernel, key rows by a correction pass), the same arithmetic with
# the key tiles corrected inside the kernel too, and the opt-in single-fp16-product
# path.
PRECISIONS = {"default": 0, "inkernel": jl.JL_PREFILL_KEYS_IN_KERNEL, "fp16": jl.JL_PREFILL_FP16}


def prefill_workspace(prec, nbytes, dev):
    """Scratch for a prefill variant (None when the key tiles are corrected in the kernel)."""
    return None if prec == "inkernel" else torch.empty(nbytes, dtype=torch.uint8, device=dev)


def run_prefill(q, k, v, *, w0, W, base, mode=jo.MODE_SELF_EXTEND, scale=0.0, prec="default"):
    """Run jl_bifocal_prefill on CPU bf16 inputs; returns (O float32 CPU, LSE CPU, dev_error)."""
    dev = torch.device("cuda")
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty_like(qd)
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)
    ws = prefill_workspace(prec, jl.jl_prefill_workspace_bytes(B, L, Hq, Hkv, D), dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    m = MODES[mode] | PRECISIONS[prec]
    jl.jl_bifocal_prefill(qd, kd, vd, o, lse, w0=w0, w_pretrained=W, rope_base=base, softmax_scale=scale,
                          mode=m, workspace=ws, dev_error=err)
    torch.cuda.synchronize()
    return o.float().cpu(), lse.cpu(), int(err.item())


def run_decode(q, kc, vc, *, L, w0, W, base, mode=jo.MODE_SELF_EXTEND, scale=0.0, workspace=None):
    dev = torch.device("cuda")
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    qd, kd, vd = q.to(dev), kc.to(dev), vc.to(dev)
    o = torch.empty_like(qd)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.zeros(jl.jl_decode_workspace_bytes(B, L, Hq, Hkv, D), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    jl.jl_bifocal_decode(qd, kd, vd, o, lse, L=L, w0=w0, w_pretrained=W, rope_base=base, softmax_scale=scale,
                         mode=MODES[mode], workspace=workspace, dev_error=err)
    torch.cuda.synchronize()
    return o.float().cpu(), lse.cpu(), int(err.item())


def assert_close(o_gpu, o_ref, lse_gpu, lse_ref, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    err = np.abs(o_gpu - o_ref)
    lerr = np.abs(np.asarray(lse_gpu, dtype=np.float64) - np.asarray(lse_ref, dtype=np.float64))
    msg = f"{what}: O max {err.max():.3e} mean {err.mean():.3e}; LSE max {lerr.max():.3e}"
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(lse_gpu)), msg
    assert err.max() <= O_MAX_ABS, msg
    assert err.mean() <= O_MEAN_ABS, msg
    assert lerr.max() <= LSE_MAX_ABS, msg
    return err.max(), err.mean(), lerr.max()


def sample_rows(L: int, w0: int, n: int, seed: int = 0):
    """Seeded query rows plus the band and tile edges."""
    rng = np.random.default_rng(seed)
    edges = {0, L - 1, w0 - 1, w0, w0 + 1, 127, 128, L // 2}
    for m in (1, 2, 7, L // 128 - 1, L // 128):
        edges |= {128 * m - 1, 128 * m}
    rows = set(int(x) for x in edges if 0 <= x < L)
    rows |= set(int(x) for x in rng.choice(L, size=min(n, L), replace=False))
    return np.array(sorted(rows), dtype=np.int64)


def oracle_prefill_rows(q, k, v, rows, heads, p: jo.BifocalParams):
    """Oracle rows for the listed heads (b = 0): dict h -> (O[n, d], LSE[n])."""
    Hq, Hkv = q.shape[2], k.shape[2]
    r = Hq // Hkv
    out = {}
    by_g = {}
    for h in heads:
        by_g.setdefault(h // r, []).append(h)
    for g, hs in by_g.items():
        kg = k[0, :, g, :].double().numpy()
        vg = v[0, :, g, :].double().numpy()
        for h in hs:
            qh = q[0, rows, h, :].double().numpy()
            out[h] = jo.attention_rows(qh, rows, kg, vg, p)
    return out


def block_passes(L, w0, tile=128):
    """(remote passes, local passes) of every 128-row query block: a key block
    gets a remote pass if it holds a causal pair that is not local, a local
    pass if it holds a local one (the oracle's is_local)."""
    out = []
    for a in range(-(-L // tile)):
        i = np.arange(tile * a, min(tile * a + tile, L))
        n_rem = n_loc = 0
        for c in range(a + 1):
            j = np.arange(tile * c, min(tile * c + tile, L))
            causal = i[:, None] >= j[None, :]
            loc = jo.is_local(i[:, None], j[None, :], w0)
            n_loc += bool(np.any(causal & loc))
            n_rem += bool(np.any(causal & ~loc))
        out.append((n_rem, n_loc))
    return out


# (L, w0) with W = L / 2 (G 2): query blocks of one to five passes, the switch
# from remote to local operands after pass 1, 2 or never, and blocks with only
# local passes, i.e. the first passes of a block and its last ones, where the
# prefill kernel's pipeline starts and drains
SHORT_PASS_CASES = [(128, 0), (128, 64), (256, 0), (256, 100), (256, 200), (384, 0), (384, 150), (384, 260)]
