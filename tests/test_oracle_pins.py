"""Pins for the fp64 oracle against what the Jet-Long pages and mathematics fix.

Each test pins the oracle to something other than itself: hand-evaluated
tables of the page formulas (tests/golden/), closed forms of the rotation,
library routines the special cases reduce to, an independent brute force and
the pages' own inclusion-exclusion formulation.  ``test_oracle_mutations.py``
plants plausible mistakes in the oracle and checks that these pins catch them.
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import jetlong_oracle as jo
from rope_context_extension_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [list(map(int, ln.split())) for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------------------
# Position algebra
# ---------------------------------------------------------------------------

def test_group_size_golden():
    for L, W, G in _rows("group_size.txt"):
        assert jo.group_size(L, W) == G, (L, W)


def test_positions_tiny_golden():
    G = jo.group_size(512, 128)
    for i, f, pse, pnone in _rows("positions_tiny.txt"):
        assert int(jo.key_remote_position(i, G)) == f
        assert int(jo.query_remote_position(i, G, 32, jo.MODE_SELF_EXTEND)) == pse
        assert int(jo.query_remote_position(i, G, 32, jo.MODE_NONE)) == pnone


def test_group_size_is_minimal_in_range_integer():
    # G = ceil(L/W) is the smallest integer with floor((L-1)/G) <= W-1
    # (gist.science summary §1: minimal compression keeping remote angles in range).
    for W in (1, 2, 3, 7, 128):
        for L in range(1, 6 * W + 3):
            G = jo.group_size(L, W)
            assert (L - 1) // G <= W - 1
            if G > 1:
                assert (L - 1) // (G - 1) > W - 1


@pytest.mark.parametrize("mode", [jo.MODE_NONE, jo.MODE_SELF_EXTEND])
def test_remote_relative_range_exhaustive(mode):
    for L, W, w0 in [(40, 8, 0), (40, 8, 3), (64, 16, 5), (97, 13, 11), (33, 32, 4), (50, 7, 49), (50, 7, 60)]:
        G = jo.group_size(L, W)
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        remote = (j <= i) & ~jo.is_local(i, j, w0)
        rel = jo.query_remote_position(i, G, w0, mode) - jo.key_remote_position(j, G)
        rng = jo.remote_relative_range(L, w0, W, mode)
        if not remote.any():
            assert rng is None
            continue
        assert (int(rel[remote].min()), int(rel[remote].max())) == rng
        if mode == jo.MODE_NONE:
            assert rel[remote].min() >= 0 and rel[remote].max() < W  # in the pretrained range
        else:
            assert rel[remote].min() >= w0                             # continues from w0


def test_self_extend_overshoot_is_as_computed():
    # The recorded reading's remote range at the main workloads (closed form).
    assert jo.remote_relative_range(512, 32, 128, jo.MODE_SELF_EXTEND) == (32, 151)
    assert jo.remote_relative_range(131072, 4096, 32768, jo.MODE_SELF_EXTEND) == (4096, 35839)
    assert jo.remote_relative_range(131072, 4096, 32768, jo.MODE_NONE) == (1024, 32767)


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def test_rope_d2_is_plane_rotation():
    # d = 2: one pair, theta_0 = 1, so R(p) is the plane rotation by p radians.
    x = np.array([[0.3, -1.7]])
    for p in (0, 1, 5, -3, 100003):
        c, s = math.cos(p), math.sin(p)
        want = np.array([[c * 0.3 - s * -1.7, s * 0.3 + c * -1.7]])
        np.testing.assert_allclose(jo.rope_rotate(x, p, 10000.0), want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("L,w0", [(1, 0), (5, 3), (128, 0), (129, 1), (200, 100), (300, 129), (512, 32),
                                  (640, 256), (777, 300), (1000, 1), (1024, 5000)])
def test_tile_classes_closed_form_equals_pair_enumeration(L, w0):
    # brute force over every pair of every 128 x 128 block
    assert jo.tile_classes(L, w0) == jo.tile_classes(L, w0, exhaustive=True)


def test_tile_classes_by_hand():
    # L 512, w0 32: four diagonal blocks hold distances 0..127 and the three
    # first sub-diagonal blocks 1..255, so all seven straddle the band edge;
    # the three blocks two or more apart hold distances >= 129: remote only.
    assert jo.tile_classes(512, 32) == (0, 7, 3)
    # w0 0: no local pair; w0 >= L: no remote pair (10 causal blocks at L 512)
    assert jo.tile_classes(512, 0) == (0, 0, 10)
    assert jo.tile_classes(512, 512) == (10, 0, 0)
    # w0 1: only i == j is local, so only the four diagonal blocks hold it
    assert jo.tile_classes(512, 1) == (0, 4, 6)
    # tile 1: every pair is its own block
    L, w0 = 9, 3
    n_loc = sum(1 for i in range(L) for j in range(i + 1) if i - j < w0)
    assert jo.tile_classes(L, w0, tile=1) == (n_loc, 0, L * (L + 1) // 2 - n_loc)


def test_rope_frequencies_closed_form():
    th = jo.rope_frequencies(8, 10000.0)
    np.testing.assert_allclose(th, [1.0, 0.1, 0.01, 0.001], rtol=1e-14)


def test_rope_pairs_are_half_split():
    # Only the coordinate pair (t, t + d/2) mixes; the angle of pair t is p*theta_t.
    d, base, p = 8, 10000.0, 7
    th = jo.rope_frequencies(d, base)
    for t in range(d // 2):
        e = np.zeros((1, d))
        e[0, t] = 1.0
        out = jo.rope_rotate(e, p, base)[0]
        want = np.zeros(d)
        want[t] = math.cos(p * th[t])
        want[t + d // 2] = math.sin(p * th[t])
        np.testing.assert_allclose(out, want, atol=1e-14)


def test_rope_dot_depends_on_relative_position_only():
    rng = np.random.default_rng(3)
    x, y = rng.standard_normal((2, 1, 64))
    for a, b in [(5, 2), (1000, 997), (131071, 131068)]:
        lhs = float((jo.rope_rotate(x, a, 1e6) @ jo.rope_rotate(y, b, 1e6).T)[0, 0])
        rhs = float((jo.rope_rotate(x, a - b, 1e6) @ y.T)[0, 0])
        assert abs(lhs - rhs) < 1e-9


def test_correction_rotation_composes_to_remote_position():
    # gist.science summary §2: RoPE rotations compose additively, so the
    # correction R(f(j) - j) applied to the cached base key R(j) k equals
    # R(f(j)) k; likewise for queries with p_q(i).
    rng = np.random.default_rng(4)
    k_raw = rng.standard_normal((1, 128))
    L, W, w0 = 131072, 32768, 4096
    G = jo.group_size(L, W)
    for j in (0, 1, 4095, 4096, 65537, 131071):
        cached = jo.rope_rotate(k_raw, j, 1e6)
        f = int(jo.key_remote_position(j, G))
        np.testing.assert_allclose(jo.rope_rotate(cached, f - j, 1e6), jo.rope_rotate(k_raw, f, 1e6),
                                   atol=1e-9)
        pq = int(jo.query_remote_position(j, G, w0, jo.MODE_SELF_EXTEND))
        np.testing.assert_allclose(jo.rope_rotate(cached, pq - j, 1e6), jo.rope_rotate(k_raw, pq, 1e6),
                                   atol=1e-9)


# ---------------------------------------------------------------------------
# Whole attention: reductions to library routines
# ---------------------------------------------------------------------------

def _sdpa_causal(q, k, v, scale=None):
    """Plain causal attention on already-rotated Q/K via torch SDPA in float64."""
    qd = q.double().permute(0, 2, 1, 3)  # B, Hq, L, d
    r = q.shape[2] // k.shape[2]
    kd = k.double().repeat_interleave(r, dim=2).permute(0, 2, 1, 3)
    vd = v.double().repeat_interleave(r, dim=2).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("mode", [jo.MODE_NONE, jo.MODE_SELF_EXTEND])
def test_g1_reduces_to_plain_causal_rope(mode):
    # L <= w_pretrained gives G = 1: exactly the base model (Jet-Long review, "Key idea").
    q, k, v = synthetic.prefill_inputs(1, 96, 4, 2, 32, seed=5)
    p = jo.BifocalParams(L=96, w0=17, w_pretrained=96, base=10000.0, mode=mode)
    o, _ = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    np.testing.assert_allclose(o, _sdpa_causal(q, k, v), atol=1e-12)


@pytest.mark.parametrize("mode", [jo.MODE_NONE, jo.MODE_SELF_EXTEND])
def test_w0_ge_L_reduces_to_plain_causal_rope(mode):
    q, k, v = synthetic.prefill_inputs(1, 80, 2, 1, 32, seed=6)
    p = jo.BifocalParams(L=80, w0=80, w_pretrained=16, base=10000.0, mode=mode)  # G = 5
    o, _ = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    np.testing.assert_allclose(o, _sdpa_causal(q, k, v), atol=1e-12)


def test_single_key_returns_first_value():
    q, k, v = synthetic.prefill_inputs(1, 1, 2, 1, 64, seed=7)
    p = jo.BifocalParams(L=1, w0=0, w_pretrained=128, base=10000.0)
    o, lse = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0].double().numpy(), atol=1e-15)
    np.testing.assert_allclose(o[0, 0, 1], v[0, 0, 0].double().numpy(), atol=1e-15)
    s = float(q[0, 0, 0].double() @ k[0, 0, 0].double()) / 8.0
    assert abs(lse[0, 0, 0] - s) < 1e-12


# ---------------------------------------------------------------------------
# Independent brute force on tiny inputs
# ---------------------------------------------------------------------------

def _bf_rotate(x, pos, base):
    d = len(x)
    h = d // 2
    out = [0.0] * d
    for t in range(h):
        a = pos * base ** (-2.0 * t / d)
        c, s = math.cos(a), math.sin(a)
        out[t] = x[t] * c - x[t + h] * s
        out[t + h] = x[t + h] * c + x[t] * s
    return out


def _brute_force(q, k, v, L, w0, W, base, mode):
    """Pure-Python loops over every (head, i, j): its own G, f, p_q and rotations."""
    B, _, Hq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0][0])
    G = max(1, (L + W - 1) // W)
    shift = (w0 - w0 // G) if mode == jo.MODE_SELF_EXTEND else 0
    out = {}
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(L):
                qi = _bf_rotate(q[b][i][h], -i, base)
                scores = []
                for j in range(i + 1):
                    kj = _bf_rotate(k[b][j][g], -j, base)
                    if i - j < w0:
                        a, c = _bf_rotate(qi, i, base), _bf_rotate(kj, j, base)
                    else:
                        a, c = _bf_rotate(qi, i // G + shift, base), _bf_rotate(kj, j // G, base)
                    scores.append(sum(x * y for x, y in zip(a, c)) / math.sqrt(d))
                m = max(scores)
                e = [math.exp(s - m) for s in scores]
                tot = sum(e)
                o = [sum(e[j] * v[b][j][g][t] for j in range(i + 1)) / tot for t in range(d)]
                out[(b, i, h)] = (o, m + math.log(tot))
    return out


@pytest.mark.parametrize("L,W,w0,mode", [
    (24, 8, 5, jo.MODE_SELF_EXTEND), (24, 8, 5, jo.MODE_NONE), (31, 7, 0, jo.MODE_SELF_EXTEND),
    (20, 6, 20, jo.MODE_NONE), (17, 4, 3, jo.MODE_SELF_EXTEND)])
def test_brute_force_tiny(L, W, w0, mode):
    q, k, v = synthetic.prefill_inputs(1, L, 4, 2, 8, seed=L + w0)
    base = 100.0
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=base, mode=mode)
    o, lse = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    bf = _brute_force(q.double().tolist(), k.double().tolist(), v.double().tolist(), L, w0, W, base, mode)
    for (b, i, h), (ob, lb) in bf.items():
        np.testing.assert_allclose(o[b, i, h], ob, atol=1e-12)
        assert abs(lse[b, h, i] - lb) < 1e-12


def test_brute_force_l64_tiny_shape():
    # L = 64 at the tiny workload's head shape (2 q heads / 1 kv head, d = 64).
    L, W, w0, base = 64, 16, 8, 10000.0
    q, k, v = synthetic.prefill_inputs(1, L, 2, 1, 64, seed=0)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=base)
    o, lse = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    bf = _brute_force(q.double().tolist(), k.double().tolist(), v.double().tolist(), L, w0, W, base,
                      jo.MODE_SELF_EXTEND)
    for (b, i, h), (ob, lb) in bf.items():
        np.testing.assert_allclose(o[b, i, h], ob, atol=1e-11)
        assert abs(lse[b, h, i] - lb) < 1e-11


# ---------------------------------------------------------------------------
# The pages' inclusion-exclusion formulation agrees with the direct definition
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L,W,w0,mode", [(512, 128, 32, jo.MODE_SELF_EXTEND), (512, 128, 32, jo.MODE_NONE),
                                         (300, 64, 0, jo.MODE_SELF_EXTEND), (300, 64, 299, jo.MODE_NONE),
                                         (257, 100, 64, jo.MODE_SELF_EXTEND)])
def test_inclusion_exclusion_matches_direct(L, W, w0, mode):
    q, k, v = synthetic.prefill_inputs(1, L, 2, 1, 64, seed=1, outlier_frac=0.01)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=10000.0, mode=mode)
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()
    rows = np.arange(L)
    for h in range(2):
        o1, l1 = jo.attention_rows(qn[0, :, h], rows, kn[0, :, 0], vn[0, :, 0], p)
        o2, l2 = jo.inclusion_exclusion_rows(qn[0, :, h], rows, kn[0, :, 0], vn[0, :, 0], p)
        # The merge subtracts W_C from W_B, so fp64 round-off is amplified by
        # the cancellation (worst with the x8 outlier keys): 1e-8, not 1e-12.
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-8)
        np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-8)


# ---------------------------------------------------------------------------
# Invariants and decode consistency
# ---------------------------------------------------------------------------

def test_softmax_invariants_tiny_workload():
    q, k, v = synthetic.prefill_inputs(1, 512, 2, 1, 64, seed=0)
    p = jo.BifocalParams(L=512, w0=32, w_pretrained=128, base=10000.0)
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()
    rows = np.arange(512)
    s = jo.bifocal_scores(qn[0, :, 0], rows, kn[0, :, 0], p)
    o, lse = jo.softmax_rows(s, vn[0, :, 0])
    assert np.all(lse >= s.max(axis=1) - 1e-12)                 # LSE >= max score
    assert np.all(lse <= s.max(axis=1) + np.log(rows + 1) + 1e-12)
    vmax = np.maximum.accumulate(np.abs(vn[0, :, 0]), axis=0)
    assert np.all(np.abs(o) <= vmax + 1e-12)                    # convex combination of values


@pytest.mark.parametrize("mode", [jo.MODE_NONE, jo.MODE_SELF_EXTEND])
def test_decode_equals_last_prefill_row(mode):
    L, W, w0 = 200, 64, 16
    q, k, v = synthetic.prefill_inputs(2, L, 4, 2, 32, seed=9)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=10000.0, mode=mode)
    o_pf, lse_pf = jo.prefill_dense(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    o_dec, lse_dec = jo.decode(q[:, L - 1].float().numpy(), k.float().numpy(), v.float().numpy(), p)
    np.testing.assert_allclose(o_dec, o_pf[:, L - 1], atol=1e-12)
    np.testing.assert_allclose(lse_dec, lse_pf[:, :, L - 1], atol=1e-12)


def test_decode_ignores_cache_beyond_L():
    L, W, w0 = 150, 64, 16
    q, k, v = synthetic.decode_inputs(1, 256, 4, 1, 32, seed=2)
    p = jo.BifocalParams(L=L, w0=w0, w_pretrained=W, base=10000.0)
    o1, l1 = jo.decode(q.float().numpy(), k.float().numpy(), v.float().numpy(), p)
    k2, v2 = k.clone(), v.clone()
    k2[:, L:] = 100.0
    v2[:, L:] = -100.0
    o2, l2 = jo.decode(q.float().numpy(), k2.float().numpy(), v2.float().numpy(), p)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
