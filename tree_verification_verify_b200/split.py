"""One long prefix split across ranks (one process per GPU): rank r holds
the prefix rows [lo_r, hi_r) of every sequence, computes prefix-only
partials of tree_verify_attn over them (the last rank also attends to the
tree keys), the partials are all-gathered, and tree_verify_attn_merge
combines them by log-sum-exp into the whole tree attention on every rank.
The host-side partition lives here so that every caller splits the same
way."""

from __future__ import annotations

import torch


def prefix_slice(rank: int, world: int, Lmax: int):
    """Prefix rows [lo, hi) held by `rank` of `world` for a cache of Lmax rows:
    contiguous, in rank order, sizes differing by at most one row."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    return (rank * Lmax) // world, ((rank + 1) * Lmax) // world


def slice_prefix_len(prefix_len: torch.Tensor, lo: int, hi: int) -> torch.Tensor:
    """Per-sequence prefix length inside the slice [lo, hi): the keys of a
    sequence with prefix_len L that fall in the slice, as int32."""
    return torch.clamp(prefix_len.to(torch.int64) - lo, 0, hi - lo).to(torch.int32)


def split_tree_verify_attn(q, k_slice, v_slice, prefix_len, k_tree, v_tree, parent, rank: int, world: int,
                           lo: int, hi: int, group=None, parts=None, out=None, lse=None):
    """Tree attention of a prefix split across the ranks of `group`
    (torch.distributed initialised; NCCL for CUDA tensors).  k_slice and
    v_slice are this rank's cache rows [lo, hi) ([B][hi - lo][Hkv][d]);
    prefix_len is every sequence's whole prefix length.  Returns (out, lse)
    of the whole tree attention, identical on every rank.  `parts`, when
    given, is a (part_o, part_lse, all_o, all_lse) tuple of preallocated
    buffers."""
    import tree_verification_verify_b200 as tv
    B, T, Hq, d = q.shape
    pl = slice_prefix_len(prefix_len, lo, hi)
    if parts is None:
        parts = (torch.empty_like(q), torch.empty(B, T, Hq, dtype=torch.float32, device=q.device),
                 torch.empty((world,) + tuple(q.shape), dtype=q.dtype, device=q.device),
                 torch.empty(world, B, T, Hq, dtype=torch.float32, device=q.device))
    part_o, part_l, all_o, all_l = parts
    tv.tree_verify_attn(q, k_slice, v_slice, pl, k_tree, v_tree, parent, out=part_o, lse=part_l,
                        prefix_only=(rank != world - 1))
    if world > 1:
        import torch.distributed as dist
        dist.all_gather_into_tensor(all_o, part_o, group=group)
        dist.all_gather_into_tensor(all_l, part_l, group=group)
    else:
        all_o[0].copy_(part_o)
        all_l[0].copy_(part_l)
    return tv.tree_verify_attn_merge(all_o, all_l, out=out, lse=lse)
