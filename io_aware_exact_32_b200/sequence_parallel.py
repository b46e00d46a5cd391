"""Sequence-parallel decode across ranks (one process per GPU).

Each rank holds one slice of every sequence's KV cache: rank r of W owns key positions
[r * Ls, (r + 1) * Ls) with Ls = ceil(Lmax / W), stored as a [B, H, Ls, d] cache.  A rank computes
the split-KV partials of its slice (fa_decode_partials: per split, the running max m, the sum l
and the unnormalised output), the ranks all-gather those partials, and every rank merges all
W * S of them with the same (m, l, O) recurrence that merges splits on one device
(fa_decode_merge).  That recurrence is the Flash-Decoding reduction of "Transformer、注意力机制与
优化" (section Flash-Decoding), applied once more across devices: the result is the exact
attention over the whole sequence.  The collective carries B * H * S * (d + 2) fp32 values per
rank, not the cache.
"""
from __future__ import annotations

import math


def slice_bounds(Lmax: int, rank: int, world: int) -> tuple[int, int]:
    """(first key position, capacity Ls) of rank's slice; every rank's cache has Ls rows."""
    Ls = max(1, math.ceil(Lmax / world))
    return rank * Ls, Ls


def local_lengths(seqlens, rank: int, world: int, Lmax: int):
    """Per-sequence number of valid keys in rank's slice: clamp(L_b - start, 0, Ls)."""
    start, Ls = slice_bounds(Lmax, rank, world)
    return (seqlens - start).clamp(min=0, max=Ls)


def decode_sequence_parallel(q, k_local, v_local, local_seqlens, group=None, scale=None, num_splits: int = 0,
                             stream=None, partials_fn=None, merge_fn=None):
    """Decode attention over sequences whose KV caches are split by position across the ranks of
    `group` (all ranks when None; a single process when torch.distributed is not initialised).

    q [B, H, 1, d] bf16 (the same on every rank); k_local, v_local [B, H, Ls, d] bf16 this rank's
    slice; local_seqlens [B] int32 the valid keys of the slice (local_lengths).  Returns
    (o [B, H, 1, d] bf16, lse [B, H] fp32), identical on every rank.  partials_fn / merge_fn
    default to the CUDA entry points and exist so that the host logic can be exercised without a GPU.
    """
    import torch
    import torch.distributed as dist

    from . import fa_decode_merge, fa_decode_num_splits, fa_decode_partials

    partials_fn = partials_fn or fa_decode_partials
    merge_fn = merge_fn or fa_decode_merge
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    B, H, _, d = q.shape
    S = fa_decode_num_splits(k_local.shape[2], num_splits) if partials_fn is fa_decode_partials else max(1, num_splits)
    part_o = torch.empty(B, H, S, d, dtype=torch.float32, device=q.device)
    part_ml = torch.empty(B, H, S, 2, dtype=torch.float32, device=q.device)
    partials_fn(q, k_local, v_local, local_seqlens, part_o, part_ml, scale=scale, num_splits=num_splits,
                stream=stream)
    if world > 1:
        # Gathered along the first dimension ([world * B, ...]), viewed as [world, B, ...].
        all_o = torch.empty(world * B, H, S, d, dtype=torch.float32, device=q.device)
        all_ml = torch.empty(world * B, H, S, 2, dtype=torch.float32, device=q.device)
        dist.all_gather_into_tensor(all_o, part_o, group=group)
        dist.all_gather_into_tensor(all_ml, part_ml, group=group)
        all_o, all_ml = all_o.view(world, B, H, S, d), all_ml.view(world, B, H, S, 2)
    else:
        all_o, all_ml = part_o.unsqueeze(0), part_ml.unsqueeze(0)
    o = torch.empty(B, H, 1, d, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(B, H, dtype=torch.float32, device=q.device)
    merge_fn(all_o, all_ml, o, lse, stream=stream)
    return o, lse
