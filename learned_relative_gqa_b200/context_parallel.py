"""Context-parallel (sequence-sharded) learned-relative GQA attention.

Each rank of a process group holds one contiguous slice of the sequence, the
same slice on the query and on the key side: its query rows
[r * S_loc, (r + 1) * S_loc) with their q, profiles, sink, valid and positions,
and the keys of those tokens (k, v, key_valid, key_positions). Ranks hold
slices in rank order.

* forward: the key-side tensors of every rank are all-gathered along the
  sequence (NCCL over NVLink between GPUs; the copies land in this GPU's own
  memory, so the attention kernels read only local memory), then the
  single-GPU kernels run the local queries against the global keys with
  ``query_offset = r * S_loc``;
* backward: the keys are gathered again, the local queries' contributions to
  the gradient of every key are computed, and dK / dV are reduce-scattered so
  that each rank receives the gradient of its own key slice; dQ, dprofiles and
  dsink belong to the local queries and stay local.

The split into a local query slice at ``query_offset`` against global keys and
key-side masks is the one the NeMo AutoModel page for
``Inkling2FlexAttention.forward`` describes for its ``query_offset``,
``key_valid`` and ``key_positions`` arguments (context-parallel attention).
The attention itself is the C-ABI library (``binding.forward`` /
``binding.backward``); ``attn_forward`` / ``attn_backward`` let a caller supply
another implementation with the same signature.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def _group_info(group):
    return dist.get_world_size(group), dist.get_rank(group)


def gather_sequence(t: torch.Tensor, group=None) -> torch.Tensor:
    """[B, S_loc, ...] on every rank -> [B, world * S_loc, ...] in rank order."""
    world, _ = _group_info(group)
    t = t.contiguous()
    if world == 1:
        return t
    is_bool = t.dtype == torch.bool
    src = t.to(torch.uint8) if is_bool else t  # not every backend moves bool tensors
    parts = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(parts, src, group=group)
    g = torch.cat(parts, dim=1)
    return g.bool() if is_bool else g


def reduce_scatter_sequence(t: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of [B, world * S_loc, ...] over the ranks, this rank's slice [B, S_loc, ...]."""
    world, rank = _group_info(group)
    if world == 1:
        return t.contiguous()
    chunks = [c.contiguous() for c in t.chunk(world, dim=1)]
    if dist.get_backend(group) == "nccl":
        out = torch.empty_like(chunks[rank])
        dist.reduce_scatter(out, chunks, group=group)
        return out
    # backends without reduce-scatter: all-reduce, keep the own slice
    full = t.contiguous().clone()
    dist.all_reduce(full, group=group)
    return full.chunk(world, dim=1)[rank].contiguous()


def _key_side(q, k, v, valid, key_valid, positions, key_positions, group):
    """Global keys and key-side metadata; defaults follow the single-GPU API
    (key_valid defaults to all valid, key_positions to the local positions)."""
    if key_valid is None:
        key_valid = torch.ones(k.shape[:2], dtype=valid.dtype, device=valid.device)
    if key_positions is None:
        if positions is None:
            raise ValueError("context-parallel attention needs explicit positions")
        key_positions = positions
    return (gather_sequence(k, group), gather_sequence(v, group), gather_sequence(key_valid, group),
            gather_sequence(key_positions, group))


def forward(q, k, v, profiles, sink, valid, key_valid=None, positions=None, key_positions=None, *,
            window: int = 0, group=None, attn_forward: Optional[Callable] = None):
    """Local out [B, S_loc, Hq, D] and lse [B, S_loc, Hq] of the local query slice."""
    _, rank = _group_info(group)
    if positions is None:
        raise ValueError("context-parallel attention needs explicit positions")
    kg, vg, kvg, kpg = _key_side(q, k, v, valid, key_valid, positions, key_positions, group)
    if attn_forward is None:
        from learned_relative_gqa_b200 import binding
        attn_forward = binding.forward
    return attn_forward(q, kg, vg, profiles, sink, valid, kvg, positions, kpg, window=window,
                        query_offset=rank * q.shape[1])


def backward(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout, dlse=None, *,
             window: int = 0, group=None, attn_backward: Optional[Callable] = None):
    """dict dq, dprofiles, dsink (local queries) and dk, dv (local key slice, summed over ranks)."""
    _, rank = _group_info(group)
    if positions is None:
        raise ValueError("context-parallel attention needs explicit positions")
    kg, vg, kvg, kpg = _key_side(q, k, v, valid, key_valid, positions, key_positions, group)
    if attn_backward is None:
        from learned_relative_gqa_b200 import binding
        attn_backward = binding.backward
    g = attn_backward(q, kg, vg, profiles, sink, valid, kvg, positions, kpg, out, lse, dout, dlse, window=window,
                      query_offset=rank * q.shape[1])
    g = dict(g)
    g["dk"] = reduce_scatter_sequence(g["dk"], group)
    g["dv"] = reduce_scatter_sequence(g["dv"], group)
    return g
