"""Context-parallel (sequence-sharded) learned-relative GQA attention.

Each rank of a process group holds one contiguous slice of the sequence, the
same slice on the query and on the key side: its query rows
[r * S_loc, (r + 1) * S_loc) with their q, profiles, sink, valid and positions,
and the keys of those tokens (k, v, key_valid, key_positions). Ranks hold
slices in rank order.

* forward: the key-side tensors of every rank are all-gathered along the
  sequence (NCCL over NVLink between GPUs; the copies land in this GPU's own
  memory, so the attention kernels read only local memory). The gather is
  started asynchronously and, while it is in flight, the local queries are run
  against the local keys (the diagonal block, sink included). Once the gather
  completes, the local queries are run against the keys of the ranks before
  this one (``query_offset = r * S_loc``, sink -inf: the sink is counted once),
  and the two partial results are merged by their log-sum-exps
  (``inkling_rel_attn_merge``). Keys after the slice are never visible
  (causality), so nothing else is needed.
* backward: the single-GPU backward of the local queries against the global
  keys (the forward's gathered keys when the caller passes them back, else a
  new gather), then dK / dV are reduce-scattered so that each rank receives the
  gradient of its own key slice; dQ, dprofiles and dsink belong to the local
  queries and stay local.

The split into a local query slice at ``query_offset`` against global keys and
key-side masks is the one the NeMo AutoModel page for
``Inkling2FlexAttention.forward`` describes for its ``query_offset``,
``key_valid`` and ``key_positions`` arguments (context-parallel attention);
``Inkling2Attention.setup_cp_attention`` has the model move the keys itself.
The attention is the C-ABI library (``binding.forward`` / ``binding.backward``
/ ``binding.inkling_rel_attn_merge``); ``attn_forward``, ``attn_backward`` and
``merge`` let a caller supply other implementations with the same signatures.
"""
from __future__ import annotations

from typing import Callable, NamedTuple, Optional

import torch
import torch.distributed as dist


class GatheredKeys(NamedTuple):
    """The key side of the whole sequence on this rank: k, v [B, Skv, Hkv, D],
    key_valid [B, Skv], key_positions [B, Skv]."""
    k: torch.Tensor
    v: torch.Tensor
    key_valid: torch.Tensor
    key_positions: torch.Tensor


def _group_info(group):
    return dist.get_world_size(group), dist.get_rank(group)


class _PendingGather:
    """All-gathers along dim 1, started asynchronously; ``wait()`` returns the
    concatenated tensors (rank order)."""

    def __init__(self, tensors, group):
        world, _ = _group_info(group)
        self.world = world
        self.items = []
        for t in tensors:
            t = t.contiguous()
            is_bool = t.dtype == torch.bool
            src = t.to(torch.uint8) if is_bool else t  # not every backend moves bool tensors
            if world == 1:
                self.items.append((is_bool, [src], None))
                continue
            parts = [torch.empty_like(src) for _ in range(world)]
            work = dist.all_gather(parts, src, group=group, async_op=True)
            self.items.append((is_bool, parts, work))

    def wait(self):
        out = []
        for is_bool, parts, work in self.items:
            if work is not None:
                work.wait()
            g = parts[0] if len(parts) == 1 else torch.cat(parts, dim=1)
            out.append(g.bool() if is_bool else g)
        return out


def gather_sequence(t: torch.Tensor, group=None) -> torch.Tensor:
    """[B, S_loc, ...] on every rank -> [B, world * S_loc, ...] in rank order."""
    return _PendingGather([t], group).wait()[0]


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


def _key_side_defaults(valid, key_valid, positions, key_positions):
    """Defaults of the single-GPU API: key_valid = valid, key_positions = positions."""
    if positions is None:
        raise ValueError("context-parallel attention needs explicit positions")
    return (valid if key_valid is None else key_valid), (positions if key_positions is None else key_positions)


def _library_merge(out, lse, out_part, lse_part):
    from learned_relative_gqa_b200 import binding
    binding.inkling_rel_attn_merge(out, lse, out_part, lse_part)
    return out, lse


def forward_shard(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, *, rank: int,
                  gathered: Callable[[], GatheredKeys], window: int = 0, attn_forward: Optional[Callable] = None,
                  merge: Optional[Callable] = None):
    """One rank's forward with the communication abstracted: ``gathered()`` returns
    the global key side (blocking until it is there). The local-diagonal block is
    computed before ``gathered()`` is called, so a gather in flight overlaps it.
    Returns out [B, S_loc, Hq, D], lse [B, S_loc, Hq] and the gathered keys."""
    if attn_forward is None:
        from learned_relative_gqa_b200 import binding
        attn_forward = binding.forward
    if merge is None:
        merge = _library_merge
    S_loc = q.shape[1]
    q_off = rank * S_loc
    # the diagonal block: local queries against local keys, as a problem of its own
    out, lse = attn_forward(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, window=window,
                            query_offset=0)
    keys = gathered()
    if q_off > 0:
        # the keys of the earlier ranks: every column from q_off on is masked out
        # (those keys are the diagonal block's, or lie after the slice), and the
        # sink, already counted in the diagonal block, is -inf here
        kv_prefix = keys.key_valid.clone()
        kv_prefix[:, q_off:] = 0
        no_sink = torch.full_like(sink, float("-inf"))
        out_p, lse_p = attn_forward(q, keys.k, keys.v, profiles, no_sink, valid, kv_prefix, positions,
                                    keys.key_positions, window=window, query_offset=q_off)
        out, lse = merge(out, lse, out_p, lse_p)
    return out, lse, keys


def forward(q, k, v, profiles, sink, valid, key_valid=None, positions=None, key_positions=None, *,
            window: int = 0, group=None, attn_forward: Optional[Callable] = None, merge: Optional[Callable] = None,
            return_keys: bool = False):
    """Local out [B, S_loc, Hq, D] and lse [B, S_loc, Hq] of the local query slice
    (plus the gathered keys, for the backward, with ``return_keys``)."""
    _, rank = _group_info(group)
    key_valid, key_positions = _key_side_defaults(valid, key_valid, positions, key_positions)
    pending = _PendingGather([k, v, key_valid, key_positions], group)
    out, lse, keys = forward_shard(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, rank=rank,
                                   gathered=lambda: GatheredKeys(*pending.wait()), window=window,
                                   attn_forward=attn_forward, merge=merge)
    return (out, lse, keys) if return_keys else (out, lse)


def backward(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout, dlse=None, *,
             window: int = 0, group=None, attn_backward: Optional[Callable] = None,
             keys: Optional[GatheredKeys] = None):
    """dict dq, dprofiles, dsink (local queries) and dk, dv (local key slice, summed
    over ranks). ``keys``: the forward's gathered key side (saves a gather)."""
    _, rank = _group_info(group)
    key_valid, key_positions = _key_side_defaults(valid, key_valid, positions, key_positions)
    if keys is None:
        keys = GatheredKeys(*_PendingGather([k, v, key_valid, key_positions], group).wait())
    if attn_backward is None:
        from learned_relative_gqa_b200 import binding
        attn_backward = binding.backward
    g = attn_backward(q, keys.k, keys.v, profiles, sink, valid, keys.key_valid, positions, keys.key_positions,
                      out, lse, dout, dlse, window=window, query_offset=rank * q.shape[1])
    g = dict(g)
    g["dk"] = reduce_scatter_sequence(g["dk"], group)
    g["dv"] = reduce_scatter_sequence(g["dv"], group)
    return g
