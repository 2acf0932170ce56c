"""Seeded synthetic inputs shared by the kernels' tests, the bench and the oracle.

This module only draws random numbers; it holds none of the attention or
position arithmetic.  Every tensor is drawn on the CPU from
``torch.Generator('cpu')`` so the same bytes reach the GPU path and the fp64
oracle.

Recipe (Jet-Long pages, "Validation": Qwen3 models, no released inputs):
  * ``randn`` in fp32, rounded to bf16 (round-to-nearest-even), drawn in the
    order Q, K, V (decode: q, K cache, V cache); batch elements are consecutive
    draws of the same generator.
  * Optional key outliers: a second generator (``outlier_seed``) picks
    ``outlier_frac`` of the (batch, key, kv-head) rows of K and multiplies them
    by ``outlier_scale`` (exact in bf16 for a power of two).
  * Values are read as already rotated at their absolute (base) positions,
    which leaves the N(0, 1) distribution unchanged because a rotation is
    orthogonal.
"""

from __future__ import annotations

import torch

__all__ = ["prefill_inputs", "decode_inputs", "scale_key_outliers", "outlier_rows"]


def _randn_bf16(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def outlier_rows(B: int, n: int, Hkv: int, frac: float, seed: int = 1):
    """The seeded (b, j, kv_head) index triples ``scale_key_outliers`` picks among
    the first ``n`` keys of a [B, *, Hkv, d] key tensor (three int64 tensors)."""
    total = B * n * Hkv
    count = max(1, int(round(frac * total)))
    gen = torch.Generator("cpu").manual_seed(seed)
    idx = torch.randperm(total, generator=gen)[:count]
    b = idx // (n * Hkv)
    rem = idx % (n * Hkv)
    return b, rem // Hkv, rem % Hkv


def scale_key_outliers(k: torch.Tensor, frac: float, scale: float = 8.0, seed: int = 1,
                       length: int | None = None) -> torch.Tensor:
    """Multiply a seeded ``frac`` share of the (b, j, kv_head) rows of ``k`` by ``scale``.

    ``k`` has layout [B, Lmax, Hkv, d]; rows are drawn among the first
    ``length`` keys (default all).  Returns ``k`` (modified in place).
    """
    if frac <= 0.0:
        return k
    B, Lmax, Hkv, _ = k.shape
    b, j, h = outlier_rows(B, Lmax if length is None else length, Hkv, frac, seed)
    k[b, j, h, :] = (k[b, j, h, :].float() * scale).to(torch.bfloat16)
    return k


def prefill_inputs(B: int, L: int, Hq: int, Hkv: int, d: int, seed: int = 0,
                   outlier_frac: float = 0.0, outlier_seed: int = 1):
    """Q [B, L, Hq, d], K and V [B, L, Hkv, d], bf16 on the CPU."""
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _randn_bf16(gen, (B, L, Hq, d))
    k = _randn_bf16(gen, (B, L, Hkv, d))
    v = _randn_bf16(gen, (B, L, Hkv, d))
    scale_key_outliers(k, outlier_frac, seed=outlier_seed)
    return q, k, v


def decode_inputs(B: int, Lmax: int, Hq: int, Hkv: int, d: int, seed: int = 0,
                  outlier_frac: float = 0.0, outlier_seed: int = 1, length: int | None = None):
    """q [B, Hq, d]; K and V caches [B, Lmax, Hkv, d]; bf16 on the CPU."""
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _randn_bf16(gen, (B, Hq, d))
    k = _randn_bf16(gen, (B, Lmax, Hkv, d))
    v = _randn_bf16(gen, (B, Lmax, Hkv, d))
    scale_key_outliers(k, outlier_frac, seed=outlier_seed, length=length)
    return q, k, v
