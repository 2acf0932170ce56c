"""fp64 CPU oracle for Jet-Long Dynamic Bifocal RoPE attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm may use it.  It shares no code with the CUDA
kernels; the only module both sides use is the seeded input generator
(``rope_context_extension_b200/synthetic.py``), which holds no method
arithmetic.

What it computes, and where that comes from (page titles and sections):

* Group size ``G = max(1, ceil(L / w_pretrained))`` from the *current* length
  ``L`` -- Jet-Long review (romaanj.github.io), "Method"; gist.science
  technical summary, "Methodologie §1 Dynamische Bifocale RoPE".
* Remote position map ``f(x) = floor(x / G)`` -- same two passages.
* Bifocal split: a (query i, key j) pair with relative distance ``i - j < w0``
  keeps the base RoPE score; every other causal pair is scored with remote
  positions -- Jet-Long review, "Method" (strict ``<`` is the reading adopted,
  see ``is_local``).
* Keys (and queries) arrive rotated at their absolute base positions; the
  cache is never rewritten -- Jet-Long review, "Method" ("KV cache stores
  uncompressed keys at absolute positions"); gist.science summary, "§2
  On-the-Fly Correctie Rotatie".
* Exact reduction to the base model at ``G = 1`` -- Jet-Long review, "Key idea".

Readings where the pages are silent (each is listed in the design notes):

* Query-side remote position.  ``mode="self_extend"`` (default):
  ``p_q(i) = floor(i/G) + (w0 - floor(w0/G))`` so remote relative distances
  continue from ``w0`` (the Self-Extend lineage named in the review's
  "research thread").  ``mode="none"``: ``p_q(i) = floor(i/G)``, i.e. ``f`` on
  both sides.  Both equal ``i`` at ``G = 1``.
* RoPE pairing: half-split ("rotate half") pairs ``(t, t + d/2)`` with
  ``theta_t = base ** (-2 t / d)`` (the Qwen3 family evaluated on the pages).
* ``G`` comes from the call's total ``L`` for every query row.
* Decode: ``L`` counts the cached keys including the new token, whose query
  sits at position ``L - 1``.
* Softmax scale ``1/sqrt(d)`` unless given; LSE is the natural log of the sum
  of exponentials of the scaled scores.

Everything is float64.  Rotations are built directly from ``cos``/``sin`` of
``position * theta_t``: the oracle recovers the raw vectors ``R(-i) Q_i`` and
``R(-j) K_j`` and re-rotates them to the positions each score needs.  It never
forms a correction rotation.  Library primitives used as steps: ``numpy``
``cos``/``sin``/``exp``/``log`` and matrix products.
"""

from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass

import numpy as np

MODE_NONE = "none"
MODE_SELF_EXTEND = "self_extend"
_MODES = (MODE_NONE, MODE_SELF_EXTEND)


# ---------------------------------------------------------------------------
# Position algebra (integers only)
# ---------------------------------------------------------------------------

def group_size(L: int, w_pretrained: int) -> int:
    """G = max(1, ceil(L / w_pretrained)).

    Jet-Long review, "Method"; gist.science summary, "Methodologie §1"
    (``G = max(1, ceil(L / w_pretrained))``).
    """
    if L < 0 or w_pretrained <= 0:
        raise ValueError("need L >= 0 and w_pretrained > 0")
    return max(1, -(-L // w_pretrained))


def key_remote_position(j, G: int):
    """f(j) = floor(j / G): Jet-Long review, "Method"; gist.science "§1"."""
    return np.asarray(j, dtype=np.int64) // G


def query_shift(w0: int, G: int, mode: str) -> int:
    """Constant added to floor(i/G) on the query side (reading, see header)."""
    if mode == MODE_SELF_EXTEND:
        return w0 - w0 // G
    if mode == MODE_NONE:
        return 0
    raise ValueError(f"unknown mode {mode!r}")


def query_remote_position(i, G: int, w0: int, mode: str):
    """p_q(i) = floor(i/G) + shift (reading of the unstated query-side map)."""
    return np.asarray(i, dtype=np.int64) // G + query_shift(w0, G, mode)


def is_local(i, j, w0: int):
    """Local (exact base RoPE) iff the relative distance i - j is below w0.

    Jet-Long review, "Method" ("pairs within relative distance w0 keep the
    original RoPE score"); the strict inequality is the reading adopted.
    """
    return (np.asarray(i, dtype=np.int64) - np.asarray(j, dtype=np.int64)) < w0


def remote_positions(L: int, w0: int, w_pretrained: int, mode: str):
    """(p_q(i) for i < L, f(j) for j < L) as int64 arrays."""
    G = group_size(L, w_pretrained)
    idx = np.arange(L, dtype=np.int64)
    return query_remote_position(idx, G, w0, mode), key_remote_position(idx, G)


def remote_relative_range(L: int, w0: int, w_pretrained: int, mode: str):
    """Closed-form (min, max) of p_q(i) - f(j) over remote causal pairs, or None.

    Remote pairs are j <= i with i - j >= w0.  floor(i/G) - floor(j/G) is at
    least floor((i - j)/G) >= floor(w0/G), reached at (i, j) = (w0, 0); it is
    at most floor((L-1)/G), reached at (i, j) = (L-1, 0).  Adding the query
    shift gives the range.  None when no remote pair exists (w0 > L-1).
    """
    G = group_size(L, w_pretrained)
    if L - 1 < w0:
        return None  # no remote pair exists
    s = query_shift(w0, G, mode)
    hi = (L - 1) // G + s
    lo = w0 // G + s
    return lo, hi


def tile_classes(L: int, w0: int, tile: int = 128, exhaustive: bool = False):
    """Counts of the causal tile x tile blocks of an L x L score matrix by the
    pair classes they hold: (local only, both, remote only).

    From the definitions alone: a causal pair (i, j), j <= i < L, is local iff
    ``is_local`` (i - j < w0), remote otherwise (Jet-Long review, "Method").
    Block (a, c), c <= a, holds query rows tile*a .. and keys tile*c ..; it
    holds a causal pair whenever c <= a.  ``exhaustive`` enumerates every pair
    of every block (small L); otherwise the causal distances i - j of a block,
    a contiguous integer range, are bounded by their ends: the smallest is
    max(0, tile*(a - c) - (tile - 1)) and the largest
    min(tile*a + tile - 1, L - 1) - tile*c.
    """
    if L < 1 or w0 < 0 or tile < 1:
        raise ValueError("need L >= 1, w0 >= 0, tile >= 1")
    nb = -(-L // tile)
    loc_only = both = rem_only = 0
    for a in range(nb):
        i = np.arange(tile * a, min(tile * a + tile, L), dtype=np.int64)
        for c in range(a + 1):
            if exhaustive:
                j = np.arange(tile * c, min(tile * c + tile, L), dtype=np.int64)
                dist = i[:, None] - j[None, :]
                causal = dist >= 0
                has_loc = bool(np.any(causal & (dist < w0)))
                has_rem = bool(np.any(causal & (dist >= w0)))
            else:
                dmin = max(0, tile * (a - c) - (tile - 1))
                dmax = int(i[-1]) - tile * c
                has_loc = dmin < w0
                has_rem = dmax >= w0
            if has_loc and has_rem:
                both += 1
            elif has_loc:
                loc_only += 1
            elif has_rem:
                rem_only += 1
    return loc_only, both, rem_only


# ---------------------------------------------------------------------------
# RoPE (half-split pairs), fp64
# ---------------------------------------------------------------------------

def rope_frequencies(d: int, base: float) -> np.ndarray:
    """theta_t = base ** (-2 t / d), t in [0, d/2)."""
    t = np.arange(d // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * t / d)


_CS_CACHE: dict = {}


def _cos_sin(pos, d: int, base: float):
    """cos / sin of pos * theta_t (fp64), memoised on the position values."""
    pos = np.asarray(pos, dtype=np.float64)
    key = None
    if pos.size >= 4096:
        key = (pos.shape, d, float(base), hashlib.blake2b(pos.tobytes(), digest_size=16).digest())
        hit = _CS_CACHE.get(key)
        if hit is not None:
            return hit
    ang = pos[..., None] * rope_frequencies(d, base)
    out = (np.cos(ang), np.sin(ang))
    if key is not None:
        if len(_CS_CACHE) > 16:
            _CS_CACHE.clear()
        _CS_CACHE[key] = out
    return out


def rope_rotate(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate rows of x (..., d) to integer positions ``pos`` (broadcast on ...).

    Pair t is (x[t], x[t + d/2]); rotation by angle pos * theta_t:
      x'[t]       = x[t] cos - x[t + d/2] sin
      x'[t + d/2] = x[t + d/2] cos + x[t] sin
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    c, s = _cos_sin(pos, d, base)
    lo, hi = x[..., :h], x[..., h:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


# ---------------------------------------------------------------------------
# Attention rows from the definition
# ---------------------------------------------------------------------------

@dataclass
class BifocalParams:
    L: int
    w0: int
    w_pretrained: int
    base: float
    scale: float | None = None
    mode: str = MODE_SELF_EXTEND

    def resolved_scale(self, d: int) -> float:
        return 1.0 / math.sqrt(d) if not self.scale else float(self.scale)


def rotated_keys(k: np.ndarray, p: BifocalParams):
    """(R(j) k_raw_j, R(f(j)) k_raw_j) for base-rotated keys k (L, d), fp64."""
    k = np.asarray(k, dtype=np.float64)
    G = group_size(p.L, p.w_pretrained)
    j = np.arange(k.shape[0], dtype=np.int64)
    k_hat = rope_rotate(k, -j, p.base)               # raw key vectors
    return rope_rotate(k_hat, j, p.base), rope_rotate(k_hat, key_remote_position(j, G), p.base)


def bifocal_scores(q_rows: np.ndarray, q_pos: np.ndarray, k: np.ndarray,
                   p: BifocalParams, keys=None) -> np.ndarray:
    """Scaled bifocal scores for query rows against keys 0..L-1 (fp64).

    q_rows: (n, d) base-rotated queries at absolute positions q_pos (n,).
    k:      (L, d) base-rotated keys at positions 0..L-1.
    keys:   optional ``rotated_keys(k, p)`` (the same values, computed once).
    Returns (n, L) with -inf on non-causal pairs (j > i).
    """
    n, d = q_rows.shape
    L = k.shape[0]
    G = group_size(p.L, p.w_pretrained)
    j = np.arange(L, dtype=np.int64)
    i = np.asarray(q_pos, dtype=np.int64)
    k_loc, k_rem = rotated_keys(k, p) if keys is None else (keys[0][:L], keys[1][:L])
    q_hat = rope_rotate(q_rows, -i, p.base)          # raw query vectors
    q_loc = rope_rotate(q_hat, i, p.base)
    q_rem = rope_rotate(q_hat, query_remote_position(i, G, p.w0, p.mode), p.base)
    s_loc = q_loc @ k_loc.T
    s_rem = q_rem @ k_rem.T
    local = is_local(i[:, None], j[None, :], p.w0)
    causal = j[None, :] <= i[:, None]
    s = np.where(local, s_loc, s_rem) * p.resolved_scale(d)
    return np.where(causal, s, -np.inf)


def softmax_rows(s: np.ndarray, v: np.ndarray):
    """O = softmax(s) @ v and LSE = log sum exp(s), max-shifted, fp64."""
    m = np.max(s, axis=1, keepdims=True)
    p = np.exp(s - m)
    l = np.sum(p, axis=1, keepdims=True)
    o = (p @ np.asarray(v, dtype=np.float64)) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def attention_rows(q_rows, q_pos, k, v, p: BifocalParams, chunk: int = 64):
    """O (n, d) and LSE (n,) for query rows against keys/values 0..L-1."""
    q_rows = np.asarray(q_rows, dtype=np.float64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kmax_all = int(q_pos.max()) + 1
    keys = rotated_keys(k[:kmax_all], p)
    outs, lses = [], []
    for a in range(0, q_rows.shape[0], chunk):
        qp = q_pos[a:a + chunk]
        kmax = int(qp.max()) + 1                      # keys beyond the last row are masked
        s = bifocal_scores(q_rows[a:a + chunk], qp, k[:kmax], p, keys=keys)
        o, lse = softmax_rows(s, v[:kmax])
        outs.append(o)
        lses.append(lse)
    return np.concatenate(outs, 0), np.concatenate(lses, 0)


def prefill(q, k, v, p: BifocalParams, rows=None, heads=None, batches=None):
    """Bifocal causal prefill.

    q: [B, L, Hq, d], k/v: [B, L, Hkv, d] (any array-like; widened to fp64).
    Returns dict keyed by (b, h) -> (rows, O[n, d], LSE[n]) for the requested
    rows (default: all L rows), heads (default all) and batches (default all).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    r = Hq // Hkv
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    out = {}
    for b in (range(B) if batches is None else batches):
        for h in (range(Hq) if heads is None else heads):
            g = h // r
            o, lse = attention_rows(q[b, rows, h, :], rows, k[b, :, g, :], v[b, :, g, :], p)
            out[(b, h)] = (rows, o, lse)
    return out


def prefill_dense(q, k, v, p: BifocalParams):
    """Full prefill: O [B, L, Hq, d] and LSE [B, Hq, L] (small sizes only)."""
    q = np.asarray(q, dtype=np.float64)
    B, L, Hq, d = q.shape
    o = np.zeros((B, L, Hq, d))
    lse = np.zeros((B, Hq, L))
    for (b, h), (rows, ob, lb) in prefill(q, k, v, p).items():
        o[b, rows, h, :] = ob
        lse[b, h, rows] = lb
    return o, lse


def decode(q, k_cache, v_cache, p: BifocalParams):
    """One new query per sequence at position L-1 against cache keys 0..L-1.

    q: [B, Hq, d] rotated at L-1; caches [B, Lmax, Hkv, d].
    Returns O [B, Hq, d] and LSE [B, Hq] (fp64).
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = np.shape(k_cache)[2]
    r = Hq // Hkv
    L = p.L
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for g in range(Hkv):
            kb = np.asarray(k_cache[b, :L, g, :], dtype=np.float64)
            vb = np.asarray(v_cache[b, :L, g, :], dtype=np.float64)
            heads = list(range(g * r, (g + 1) * r))
            ob, lb = attention_rows(q[b, heads, :], np.full(r, L - 1), kb, vb, p)
            o[b, heads] = ob
            lse[b, heads] = lb
    return o, lse


def decode_key_range(q, k_cache, v_cache, p: BifocalParams, key_begin: int, key_end: int):
    """Decode (query at p.L - 1) restricted to keys [key_begin, key_end).

    The scores are the definition's (``bifocal_scores`` with G from p.L); only
    the softmax is taken over the sub-range, giving that range's normalised
    output and LSE (the partial result of a sequence-split decode).
    q: [B, Hq, d]; caches [B, >= p.L, Hkv, d].  Returns O [B, Hq, d], LSE [B, Hq].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = np.shape(k_cache)[2]
    r = Hq // Hkv
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for g in range(Hkv):
            kb = np.asarray(k_cache[b, :p.L, g, :], dtype=np.float64)
            vb = np.asarray(v_cache[b, key_begin:key_end, g, :], dtype=np.float64)
            heads = list(range(g * r, (g + 1) * r))
            s = bifocal_scores(q[b, heads, :], np.full(r, p.L - 1), kb, p)[:, key_begin:key_end]
            ob, lb = softmax_rows(s, vb)
            o[b, heads] = ob
            lse[b, heads] = lb
    return o, lse


# ---------------------------------------------------------------------------
# Second formulation: inclusion-exclusion merge of three masked softmaxes
# ---------------------------------------------------------------------------

def inclusion_exclusion_parts(q_rows, q_pos, k, v, p: BifocalParams):
    """The three calls of the pages' formulation, each a masked softmax.

    Jet-Long review, "Method": (A) sliding window with base RoPE, (B) full
    causal with remote RoPE, (C) sliding window with remote RoPE.  The window
    is the local band of ``is_local`` (keys with i - j < w0).  Returns
    ((O_A, LSE_A), (O_B, LSE_B), (O_C, LSE_C)); a row with no key in a call
    has O = 0, LSE = -inf there.  Written independently of ``bifocal_scores``
    as a cross-check.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, d = q_rows.shape
    L = k.shape[0]
    G = group_size(p.L, p.w_pretrained)
    sc = p.resolved_scale(d)
    i = np.asarray(q_pos, dtype=np.int64)
    j = np.arange(L, dtype=np.int64)
    # raw vectors, then the two position assignments
    qr = rope_rotate(q_rows, -i, p.base)
    kr = rope_rotate(k, -j, p.base)
    base_s = rope_rotate(qr, i, p.base) @ rope_rotate(kr, j, p.base).T * sc
    pq = query_remote_position(i, G, p.w0, p.mode)
    fk = key_remote_position(j, G)
    rem_s = rope_rotate(qr, pq, p.base) @ rope_rotate(kr, fk, p.base).T * sc
    causal = j[None, :] <= i[:, None]
    window = causal & ((i[:, None] - j[None, :]) < p.w0)

    def masked(s, mask):
        s = np.where(mask, s, -np.inf)
        m = np.max(s, axis=1)
        ok = np.isfinite(m)
        msafe = np.where(ok, m, 0.0)
        e = np.exp(s - msafe[:, None])
        l = e.sum(axis=1)
        o = np.where(ok[:, None], (e @ v) / np.where(ok, l, 1.0)[:, None], 0.0)
        lse = np.where(ok, msafe + np.log(np.where(ok, l, 1.0)), -np.inf)
        return o, lse

    return masked(base_s, window), masked(rem_s, causal), masked(rem_s, window)


def inclusion_exclusion_rows(q_rows, q_pos, k, v, p: BifocalParams):
    """The pages' three-call formulation, merged by inclusion-exclusion.

    Jet-Long review, "Method": the calls of ``inclusion_exclusion_parts``
    merged as O = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C) with LSE
    weights W_X = exp(LSE_X - max LSE).
    """
    (oa, la), (ob, lb), (oc, lc) = inclusion_exclusion_parts(q_rows, q_pos, k, v, p)
    mm = np.maximum(np.maximum(la, lb), lc)
    wa, wb, wc = np.exp(la - mm), np.exp(lb - mm), np.exp(lc - mm)
    den = wa + wb - wc
    o = (wa[:, None] * oa + wb[:, None] * ob - wc[:, None] * oc) / den[:, None]
    return o, mm + np.log(den)
