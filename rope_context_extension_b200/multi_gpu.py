"""Multi-GPU layouts of the bifocal decode: one process per GPU.

* Head sharding: each rank owns a contiguous group of KV heads (and their query
  heads) and runs prefill / decode on it alone (head_shard_prefill /
  head_shard_decode); no data crosses GPUs unless the caller asks for every
  head's output in one place (one all-gather).
* Sequence split: each rank holds a contiguous key range of every sequence's
  cache.  Positions, G and the band come from the global length, so the base
  keys never move; each rank computes its range's partial (O, LSE) with
  jl_bifocal_decode_range, the partials are all-gathered (one collective,
  ~16 KB per rank at B 1 / 32 heads / d 128) and merged by jl_decode_combine.

torch.distributed is plumbing here (the all-gather); the arithmetic runs in the
library's kernels.  `partial_fn` / `combine_fn` can be replaced, which lets the
gather logic be exercised on CPU ranks.
"""

from __future__ import annotations


def shard_range(total: int, rank: int, world: int):
    """Contiguous split of [0, total) into `world` near-equal parts: (begin, count) of `rank`."""
    begin = (total * rank) // world
    end = (total * (rank + 1)) // world
    return begin, end - begin


def head_shard(Hkv: int, rank: int, world: int):
    """KV heads [begin, begin + count) of `rank` for head-sharded attention."""
    if Hkv % world:
        raise ValueError("the KV heads must divide evenly over the ranks")
    n = Hkv // world
    return rank * n, n


def head_shard_slices(Hq: int, Hkv: int, rank: int, world: int):
    """(kv_begin, kv_count, q_begin, q_count) of `rank`: its KV heads and the query
    heads that read them (query head h uses KV head h // (Hq / Hkv))."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    kb, kc = head_shard(Hkv, rank, world)
    r = Hq // Hkv
    return kb, kc, kb * r, kc * r


def take_heads(x, begin: int, count: int, dim: int = 2):
    """This rank's heads of a [..., heads, ...] tensor as a contiguous tensor of its own."""
    return x.narrow(dim, begin, count).contiguous()


def _gather_heads(x_r, head_dim: int, group):
    """All-gather of per-rank head shards along `head_dim` (rank-major, so rank r's
    heads land at [r * n, (r + 1) * n), matching head_shard)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = torch.empty((world,) + tuple(x_r.shape), dtype=x_r.dtype, device=x_r.device)
    dist.all_gather_into_tensor(parts.view((world * x_r.shape[0],) + tuple(x_r.shape[1:])), x_r.contiguous(),
                                group=group)
    # [world, ..., n, ...] -> [..., world * n, ...]
    moved = parts.movedim(0, head_dim)
    shape = list(x_r.shape)
    shape[head_dim] *= world
    return moved.reshape(shape)


def _default_prefill(q, k, v, kw):
    import torch
    from . import jetlong as jl
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=q.device)
    ws = kw.pop("workspace", None)
    if ws is None:
        ws = torch.empty(jl.jl_prefill_workspace_bytes(B, L, Hq, Hkv, D), dtype=torch.uint8, device=q.device)
    jl.jl_bifocal_prefill(q, k, v, o, lse, workspace=ws, **kw)
    return o, lse


def _default_decode(q, kc, vc, kw):
    import torch
    from . import jetlong as jl
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    ws = kw.pop("workspace", None)
    if ws is None:
        ws = torch.zeros(jl.jl_decode_workspace_bytes(B, kw["L"], Hq, Hkv, D), dtype=torch.uint8, device=q.device)
    jl.jl_bifocal_decode(q, kc, vc, o, lse, workspace=ws, **kw)
    return o, lse


def head_shard_prefill(q_r, k_r, v_r, *, group=None, gather: bool = False, prefill_fn=None, **kw):
    """Bifocal prefill of this rank's KV-head group.

    q_r [B, L, Hq / world, D], k_r / v_r [B, L, Hkv / world, D] hold the rank's
    heads (take_heads of the full tensors, with the ranges of head_shard_slices);
    the group is an independent problem with the same GQA ratio, G and band, so
    the kernels run on it unchanged and nothing crosses GPUs.  Returns the rank's
    (o [B, L, Hq / world, D], lse [B, Hq / world, L]); with gather=True the
    all-ranks result (o [B, L, Hq, D], lse [B, Hq, L]) on every rank instead (one
    all-gather each, only when the caller needs every head in one place).
    Keyword arguments go to jl_bifocal_prefill (w0, w_pretrained, rope_base, ...).
    """
    import torch.distributed as dist
    o_r, lse_r = (prefill_fn or _default_prefill)(q_r, k_r, v_r, dict(kw))
    if not gather or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return o_r, lse_r
    return _gather_heads(o_r, 2, group), _gather_heads(lse_r, 1, group)


def head_shard_decode(q_r, kc_r, vc_r, *, group=None, gather: bool = False, decode_fn=None, **kw):
    """Bifocal decode of this rank's KV-head group: q_r [B, Hq / world, D], caches
    [B, Lmax, Hkv / world, D].  Returns the rank's (o [B, Hq / world, D], lse
    [B, Hq / world]) or, with gather=True, every head's on every rank.  Keyword
    arguments go to jl_bifocal_decode (L, w0, w_pretrained, rope_base, ...)."""
    import torch.distributed as dist
    o_r, lse_r = (decode_fn or _default_decode)(q_r, kc_r, vc_r, dict(kw))
    if not gather or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return o_r, lse_r
    return _gather_heads(o_r, 1, group), _gather_heads(lse_r, 1, group)


def _default_partial(q, k_shard, v_shard, key_offset, key_count, total_len, kw):
    import torch
    from . import jetlong as jl
    B, Hq, D = q.shape
    Hkv = k_shard.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    ws = kw.pop("workspace", None)
    if ws is None:
        ws = torch.zeros(jl.jl_decode_workspace_bytes(B, key_count, Hq, Hkv, D), dtype=torch.uint8, device=q.device)
    jl.jl_bifocal_decode_range(q, k_shard, v_shard, o, lse, key_offset=key_offset, key_count=key_count,
                               total_len=total_len, workspace=ws, **kw)
    return o, lse


def _default_combine(o_parts, lse_parts):
    import torch
    from . import jetlong as jl
    _, B, Hq, D = o_parts.shape
    o = torch.empty(B, Hq, D, dtype=o_parts.dtype, device=o_parts.device)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=o_parts.device)
    jl.jl_decode_combine(o_parts, lse_parts, o, lse)
    return o, lse


def sequence_split_decode(q, k_shard, v_shard, *, key_offset: int, key_count: int, total_len: int, group=None,
                          partial_fn=None, combine_fn=None, **kw):
    """Decode one query per sequence whose cache is split by key range over the ranks of `group`.

    q [B, Hq, D] (rotated at total_len - 1) is the same on every rank; k_shard /
    v_shard hold this rank's key range (rows 0 .. key_count - 1 = positions
    key_offset .. key_offset + key_count - 1).  Returns (o, lse) on every rank.
    """
    import torch
    import torch.distributed as dist
    partial_fn = partial_fn or _default_partial
    combine_fn = combine_fn or _default_combine
    o_r, lse_r = partial_fn(q, k_shard, v_shard, key_offset, key_count, total_len, dict(kw))
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return combine_fn(o_r.unsqueeze(0).contiguous(), lse_r.unsqueeze(0).contiguous())
    # gathered along dim 0 (rank-major), then viewed as [world, B, ...]
    o_parts = torch.empty((world * o_r.shape[0],) + tuple(o_r.shape[1:]), dtype=o_r.dtype, device=o_r.device)
    lse_parts = torch.empty((world * lse_r.shape[0],) + tuple(lse_r.shape[1:]), dtype=lse_r.dtype,
                            device=lse_r.device)
    dist.all_gather_into_tensor(o_parts, o_r.contiguous(), group=group)
    dist.all_gather_into_tensor(lse_parts, lse_r.contiguous(), group=group)
    return combine_fn(o_parts.view((world,) + tuple(o_r.shape)), lse_parts.view((world,) + tuple(lse_r.shape)))
