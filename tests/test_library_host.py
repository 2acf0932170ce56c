"""Host-side checks of the C-ABI library (no GPU needed).

The shared library must load, export every entry point include/jl_api.h
declares, compute the integer position algebra bit-exactly against the
oracle, and reject bad arguments with the documented status codes before any
device work is launched.
"""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import jetlong as jl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jl_api.h")

JL_OK, JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_ALIGNMENT, JL_ERR_WORKSPACE = 0, -1, -2, -3, -4


@pytest.fixture(scope="module")
def lib():
    from rope_context_extension_b200 import build
    build.build()
    return jl.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(jl_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("jl_group_size", "jl_bifocal_prefill", "jl_bifocal_decode", "jl_remote_positions",
                 "jl_prefill_workspace_bytes", "jl_decode_workspace_bytes"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(jl.EXPORTED_SYMBOLS)


def test_group_size_matches_oracle(lib):
    for L in [0, 1, 127, 128, 129, 512, 16384, 32767, 32768, 32769, 49152, 65536, 65537, 100003, 131072, 131073]:
        for W in (1, 128, 32768):
            assert jl.jl_group_size(L, W) == jo.group_size(L, W)


def test_group_size_rejects_bad_args(lib):
    g = ctypes.c_int64(0)
    assert lib.jl_group_size(-1, 10, ctypes.byref(g)) == JL_ERR_INVALID_ARG
    assert lib.jl_group_size(10, 0, ctypes.byref(g)) == JL_ERR_INVALID_ARG
    assert lib.jl_group_size(10, 10, None) == JL_ERR_INVALID_ARG


@pytest.mark.parametrize("mode", [jl.JL_QSHIFT_NONE, jl.JL_QSHIFT_SELF_EXTEND])
@pytest.mark.parametrize("L,w0,W", [(512, 32, 128), (1, 0, 5), (1000, 0, 300), (1000, 77, 300), (4096, 4096, 1000),
                                    (131072, 4096, 32768), (100003, 4096, 32768), (32769, 0, 32768)])
def test_remote_positions_bit_exact(lib, L, w0, W, mode):
    q, k = jl.jl_remote_positions(L, w0, W, mode)
    omode = jo.MODE_NONE if mode == jl.JL_QSHIFT_NONE else jo.MODE_SELF_EXTEND
    pq, fk = jo.remote_positions(L, w0, W, omode)
    np.testing.assert_array_equal(q, pq.astype(np.int32))
    np.testing.assert_array_equal(k, fk.astype(np.int32))


TILE_CASES = [(L, w0) for L in (1, 127, 128, 129, 200, 383, 640, 777, 1000, 1300, 2049)
              for w0 in (0, 1, 31, 127, 128, 129, 300, 1000, 5000)]


@pytest.mark.parametrize("L,w0", TILE_CASES)
def test_prefill_tile_schedule_matches_pair_classes(lib, L, w0):
    # The attention kernel's tile schedule (local pass, remote pass or both per
    # 128 x 128 block) against the oracle's classification of the blocks' pairs.
    W = max(1, L // 3)
    loc, both, rem, passes = jl.jl_prefill_tile_classes(L, w0, W)
    assert passes == loc + 2 * both + rem
    if jo.group_size(L, W) == 1 or w0 >= L:
        nb = -(-L // 128)
        assert (loc, both, rem) == (nb * (nb + 1) // 2, 0, 0)  # exactly base RoPE: one local pass per block
    else:
        assert (loc, both, rem) == jo.tile_classes(L, w0)


@pytest.mark.parametrize("L,w0,W", [(131072, 4096, 32768), (65536, 4096, 32768), (512, 32, 128), (100003, 4096, 32768),
                                    (131072, 0, 32768)])
def test_prefill_tile_schedule_full_workloads(lib, L, w0, W):
    assert jl.jl_prefill_tile_classes(L, w0, W)[:3] == jo.tile_classes(L, w0)


def test_prefill_tile_classes_rejects_bad_args(lib):
    out = (ctypes.c_int64 * 4)()
    assert lib.jl_prefill_tile_classes(0, 0, 10, out) == JL_ERR_INVALID_ARG
    assert lib.jl_prefill_tile_classes(10, -1, 10, out) == JL_ERR_INVALID_ARG
    assert lib.jl_prefill_tile_classes(10, 0, 0, out) == JL_ERR_INVALID_ARG
    assert lib.jl_prefill_tile_classes(10, 0, 10, None) == JL_ERR_INVALID_ARG
    assert lib.jl_prefill_tile_classes((1 << 30) + 1, 0, 10, out) == JL_ERR_INVALID_ARG


def test_remote_positions_rejects_bad_args(lib):
    assert lib.jl_remote_positions(0, 0, 10, 1, None, None) == JL_ERR_INVALID_ARG
    assert lib.jl_remote_positions(10, -1, 10, 1, None, None) == JL_ERR_INVALID_ARG
    assert lib.jl_remote_positions(10, 0, 10, 7, None, None) == JL_ERR_INVALID_ARG
    assert lib.jl_remote_positions(10, 0, 10, 2, None, None) == JL_ERR_INVALID_ARG  # not a position-map mode


FP16, INKERNEL = jl.JL_PREFILL_FP16, jl.JL_PREFILL_KEYS_IN_KERNEL


def test_workspace_sizes(lib):
    # the larger of the default's (fp16 hi + lo key rows) and JL_PREFILL_FP16's needs
    assert jl.jl_prefill_workspace_bytes(1, 131072, 32, 8, 128) >= 2 * 131072 * (32 + 8) * 128
    assert jl.jl_prefill_workspace_bytes(1, 4096, 2, 2, 128) >= 4 * 4096 * 2 * 128
    assert jl.jl_prefill_workspace_bytes(0, 10, 1, 1, 64) == 0
    assert jl.jl_decode_workspace_bytes(8, 131072, 32, 8, 128) > 0
    assert jl.jl_decode_workspace_bytes(1, 10, 3, 2, 64) == 0  # Hq % Hkv != 0


# Fake, never dereferenced device addresses: argument checks return before any launch.
A = 0x10000


def _prefill(lib, q=A, k=A, v=A, o=A, lse=None, B=1, L=256, Hq=4, Hkv=2, D=128, w0=16, W=64, base=1e4, scale=0.0,
             mode=1, ws=A, ws_bytes=1 << 40):
    return lib.jl_bifocal_prefill(q, k, v, o, lse, B, L, Hq, Hkv, D, w0, W, base, scale, mode, ws, ws_bytes, None,
                                  None)


def _decode(lib, q=A, k=A, v=A, cache_len=256, o=A, lse=None, B=1, L=256, Hq=4, Hkv=2, D=128, w0=16, W=64,
            base=1e4, scale=0.0, mode=1, ws=A, ws_bytes=1 << 40):
    return lib.jl_bifocal_decode(q, k, v, cache_len, o, lse, B, L, Hq, Hkv, D, w0, W, base, scale, mode, ws,
                                 ws_bytes, None, None)


def test_prefill_argument_errors(lib):
    assert _prefill(lib, D=96) == JL_ERR_UNSUPPORTED
    # grid limits: 65535 query blocks of 128 rows, B <= 65535, a 32-bit CTA index
    assert _prefill(lib, L=65535 * 128 + 1, w0=0) == JL_ERR_UNSUPPORTED
    assert _prefill(lib, B=65536) == JL_ERR_UNSUPPORTED
    assert _prefill(lib, B=65535, L=65535 * 128, Hq=4, Hkv=2) == JL_ERR_UNSUPPORTED
    assert _decode(lib, B=65536) == JL_ERR_UNSUPPORTED
    assert _prefill(lib, Hq=3, Hkv=2) == JL_ERR_INVALID_ARG
    assert _prefill(lib, L=0) == JL_ERR_INVALID_ARG
    assert _prefill(lib, w0=-1) == JL_ERR_INVALID_ARG
    assert _prefill(lib, W=0) == JL_ERR_INVALID_ARG
    assert _prefill(lib, base=0.0) == JL_ERR_INVALID_ARG
    assert _prefill(lib, mode=2) == JL_ERR_INVALID_ARG    # not a flag
    assert _prefill(lib, mode=16 | 1) == JL_ERR_INVALID_ARG
    assert _prefill(lib, mode=FP16 | INKERNEL | 1) == JL_ERR_INVALID_ARG  # exclusive flags
    # the default and JL_PREFILL_FP16 need the workspace jl_prefill_workspace_bytes
    # reports (every call below fails its checks, so nothing is launched on the
    # fake addresses; JL_PREFILL_KEYS_IN_KERNEL needs no workspace, so its
    # workspace arguments are never checked and are not exercised here)
    need = lib.jl_prefill_workspace_bytes(1, 256, 4, 2, 128)
    for flag in (0, FP16):
        assert _prefill(lib, mode=flag | 1, ws_bytes=need // 3) == JL_ERR_WORKSPACE
        assert _prefill(lib, mode=flag | 1, ws=None) == JL_ERR_WORKSPACE
        assert _prefill(lib, mode=flag | 1, ws=A + 4) == JL_ERR_ALIGNMENT
    assert _prefill(lib, q=None) == JL_ERR_INVALID_ARG
    assert _prefill(lib, o=None) == JL_ERR_INVALID_ARG
    assert _prefill(lib, k=A + 8) == JL_ERR_ALIGNMENT
    assert _prefill(lib, o=A + 2) == JL_ERR_ALIGNMENT


def test_empty_inputs_are_rejected_before_any_launch(lib):
    # no batch, no head, no token: every entry point refuses, nothing launches
    assert _prefill(lib, B=0) == JL_ERR_INVALID_ARG
    assert _prefill(lib, Hq=0) == JL_ERR_INVALID_ARG
    assert _prefill(lib, Hkv=0) == JL_ERR_INVALID_ARG
    assert _decode(lib, B=0) == JL_ERR_INVALID_ARG
    assert _decode(lib, L=0) == JL_ERR_INVALID_ARG
    assert _decode(lib, Hq=0) == JL_ERR_INVALID_ARG
    assert lib.jl_decode_workspace_bytes(1, 0, 4, 2, 128) == 0
    assert lib.jl_prefill_workspace_bytes(1, 0, 4, 2, 128) == 0


def test_decode_argument_errors(lib):
    assert _decode(lib, D=80) == JL_ERR_UNSUPPORTED
    assert _decode(lib, Hq=32, Hkv=2) == JL_ERR_UNSUPPORTED  # more than 8 query heads per KV head
    assert _decode(lib, cache_len=100) == JL_ERR_INVALID_ARG  # L beyond the cache
    assert _decode(lib, Hq=5, Hkv=2) == JL_ERR_INVALID_ARG
    assert _decode(lib, v=None) == JL_ERR_INVALID_ARG
    assert _decode(lib, o=A + 2) == JL_ERR_ALIGNMENT
    assert _decode(lib, ws=None) == JL_ERR_WORKSPACE
    assert _decode(lib, ws_bytes=16) == JL_ERR_WORKSPACE


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.jl_status_string(code)


def test_prefill_chunk_argument_errors(lib):
    def chunk(q_offset=100, chunk_len=156, cache_len=256, **kw):
        a = dict(q=A, k=A, v=A, o=A, lse=None, B=1, Hq=4, Hkv=2, D=128, w0=16, W=64, base=1e4, scale=0.0, mode=1,
                 ws=A, ws_bytes=1 << 40)
        a.update(kw)
        return lib.jl_bifocal_prefill_chunk(a["q"], a["k"], a["v"], cache_len, a["o"], a["lse"], a["B"], q_offset,
                                            chunk_len, a["Hq"], a["Hkv"], a["D"], a["w0"], a["W"], a["base"],
                                            a["scale"], a["mode"], a["ws"], a["ws_bytes"], None, None)
    assert chunk(q_offset=200) == JL_ERR_INVALID_ARG       # chunk runs past the cache
    assert chunk(q_offset=-1) == JL_ERR_INVALID_ARG
    assert chunk(chunk_len=0) == JL_ERR_INVALID_ARG
    assert chunk(D=80) == JL_ERR_UNSUPPORTED
    assert chunk(k=A + 4) == JL_ERR_ALIGNMENT
    need = lib.jl_prefill_chunk_workspace_bytes(1, 100, 156, 4, 2, 128)
    assert need == jl.jl_prefill_chunk_workspace_bytes(1, 100, 156, 4, 2, 128) > 0
    assert chunk(ws_bytes=need - 1, mode=FP16 | 1) == JL_ERR_WORKSPACE
    assert chunk(ws_bytes=need // 3) == JL_ERR_WORKSPACE
    # a whole-sequence chunk needs what jl_prefill_workspace_bytes reports
    assert lib.jl_prefill_chunk_workspace_bytes(2, 0, 300, 8, 2, 64) == lib.jl_prefill_workspace_bytes(2, 300, 8, 2, 64)


def test_wait_timeout_check_argument_errors(lib):
    # rejected before any launch (no GPU needed)
    assert lib.jl_wait_timeout_check(None, 0.1, None) == JL_ERR_INVALID_ARG
    assert lib.jl_wait_timeout_check(A, 0.0, None) == JL_ERR_INVALID_ARG
    assert lib.jl_wait_timeout_check(A, 11.0, None) == JL_ERR_INVALID_ARG


def test_short_pass_sequences_cover_the_prefill_pipeline_edges():
    # The GPU parity cases of tests.gpu_helpers.SHORT_PASS_CASES must contain
    # query blocks whose pass sequences exercise the start and the end of the
    # prefill kernel's pipeline: one remote pass, one local pass, a switch
    # from remote to local operands after pass 1 and after pass 2, and two or
    # three remote passes without a switch.
    from tests.gpu_helpers import SHORT_PASS_CASES, block_passes
    seen = {bp for L, w0 in SHORT_PASS_CASES for bp in block_passes(L, w0)}
    for want in [(1, 0), (0, 1), (1, 1), (1, 2), (2, 2), (2, 0), (3, 0)]:
        assert want in seen, want
    # G 2 and w0 < L: every case runs the bifocal kernel, not the all-local one
    for L, w0 in SHORT_PASS_CASES:
        assert jo.group_size(L, L // 2) == 2 and w0 < L
