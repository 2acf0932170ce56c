"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

Every mutation below is applied with ``monkeypatch`` to the oracle module only;
the pins in ``test_oracle_pins.py`` are then run and at least one of them must
fail.  This is evidence that the pins constrain the oracle's arithmetic, not
just its shape.
"""

import numpy as np
import pytest

from oracle import jetlong_oracle as jo
import tests.test_oracle_pins as pins

ALL_PINS = [
    pins.test_group_size_golden,
    pins.test_positions_tiny_golden,
    pins.test_rope_d2_is_plane_rotation,
    pins.test_rope_frequencies_closed_form,
    pins.test_rope_pairs_are_half_split,
    pins.test_correction_rotation_composes_to_remote_position,
    lambda: pins.test_g1_reduces_to_plain_causal_rope(jo.MODE_SELF_EXTEND),
    lambda: pins.test_w0_ge_L_reduces_to_plain_causal_rope(jo.MODE_NONE),
    pins.test_single_key_returns_first_value,
    lambda: pins.test_brute_force_tiny(24, 8, 5, jo.MODE_SELF_EXTEND),
    lambda: pins.test_brute_force_tiny(31, 7, 0, jo.MODE_SELF_EXTEND),
    lambda: pins.test_inclusion_exclusion_matches_direct(257, 100, 64, jo.MODE_SELF_EXTEND),
    lambda: pins.test_remote_relative_range_exhaustive(jo.MODE_NONE),
]


def _band_le(i, j, w0):
    return (np.asarray(i) - np.asarray(j)) <= w0


def _rotate_wrong_sign(x, pos, base):
    return jo_rotate_orig(x, -np.asarray(pos), base)


def _rotate_interleaved(x, pos, base):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * jo.rope_frequencies(d, base)
    c, s = np.cos(ang), np.sin(ang)
    ev, od = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x * c[..., :1])
    out = np.broadcast_to(out, np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,))).copy()
    out[..., 0::2] = ev * c - od * s
    out[..., 1::2] = od * c + ev * s
    return out


jo_rotate_orig = jo.rope_rotate


def _scores_swapped(q_rows, q_pos, k, p, keys=None):
    # local and remote score sets exchanged
    i = np.asarray(q_pos)
    j = np.arange(k.shape[0])
    G = jo.group_size(p.L, p.w_pretrained)
    qh = jo.rope_rotate(q_rows, -i, p.base)
    kh = jo.rope_rotate(k, -j, p.base)
    s_loc = jo.rope_rotate(qh, i, p.base) @ jo.rope_rotate(kh, j, p.base).T
    s_rem = jo.rope_rotate(qh, jo.query_remote_position(i, G, p.w0, p.mode), p.base) @ \
        jo.rope_rotate(kh, jo.key_remote_position(j, G), p.base).T
    loc = jo.is_local(i[:, None], j[None, :], p.w0)
    s = np.where(loc, s_rem, s_loc) * p.resolved_scale(q_rows.shape[1])
    return np.where(j[None, :] <= i[:, None], s, -np.inf)


def _softmax_no_max_in_lse(s, v):
    o, lse = jo_softmax_orig(s, v)
    return o, lse - np.max(s, axis=1)


jo_softmax_orig = jo.softmax_rows

MUTATIONS = {
    "band uses <= instead of <": ("is_local", _band_le),
    "key map ceil instead of floor": ("key_remote_position", lambda j, G: -(-np.asarray(j) // G)),
    "query shift sign flipped": ("query_shift",
                                 lambda w0, G, mode: (w0 + w0 // G) if mode == jo.MODE_SELF_EXTEND else 0),
    "group size floor instead of ceil": ("group_size", lambda L, W: max(1, L // W)),
    "rotation sign flipped": ("rope_rotate", _rotate_wrong_sign),
    "interleaved instead of half-split pairs": ("rope_rotate", _rotate_interleaved),
    "frequencies use d instead of 2t/d": ("rope_frequencies",
                                          lambda d, base: np.power(float(base), -np.arange(d // 2) / d)),
    "local/remote score sets swapped": ("bifocal_scores", _scores_swapped),
    "LSE drops the max shift": ("softmax_rows", _softmax_no_max_in_lse),
    "scale dropped": ("BifocalParams.resolved_scale", lambda self, d: 1.0),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    jo._CS_CACHE.clear()  # memoised angles must not hide a planted mistake
    monkeypatch.setattr(jo, "_CS_CACHE", {})
    if attr.startswith("BifocalParams."):
        monkeypatch.setattr(jo.BifocalParams, attr.split(".")[1], fn)
    else:
        monkeypatch.setattr(jo, attr, fn)
    caught = []
    for pin in ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(getattr(pin, "__name__", "lambda"))
    assert caught, f"no pin caught the mutation: {name}"
