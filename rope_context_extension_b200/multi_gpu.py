"""Multi-GPU layouts of the bifocal decode: one process per GPU.

* Head sharding: each rank owns a contiguous group of KV heads (and their query
  heads) and runs prefill / decode on it alone; no data crosses GPUs.
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
