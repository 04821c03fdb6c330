"""Dense FP64 torch formulation used only to pin the oracle.

It restates the method differently from the oracle on purpose:

* documents are identified by ids built from position resets (a new document
  starts at every valid column whose position is 0, and at the first valid
  column), instead of the oracle's "position difference equals column
  difference" test;
* the relative distance is the column difference i_g - j (equal to the
  logical-position difference inside a document);
* the softmax, log-sum-exp and attention products are delegated to torch
  library routines (``scaled_dot_product_attention``, ``logsumexp``, autograd).

So a dropped term, a wrong sign or a transposed index in either
implementation makes the two disagree.
"""
from __future__ import annotations

import torch


def doc_ids(valid: torch.Tensor, positions: torch.Tensor) -> torch.Tensor:
    """[B,T] document ids (-1 on invalid columns) from position resets."""
    B, T = valid.shape
    ids = torch.full((B, T), -1, dtype=torch.int64)
    for b in range(B):
        cur = -1
        started = False
        for t in range(T):
            if not bool(valid[b, t]):
                continue
            if not started or int(positions[b, t]) == 0:
                cur += 1
                started = True
            ids[b, t] = cur
    return ids


def allowed_mask(valid, key_valid, positions, key_positions, *, window: int, query_offset: int = 0,
                 heads_q: int) -> torch.Tensor:
    """Boolean [B,Hq,S,Skv] mask of allowed (query, key) pairs."""
    B, S = valid.shape
    Skv = key_valid.shape[1]
    kid = doc_ids(key_valid, key_positions)
    # the query side is the slice [query_offset, query_offset + S) of the key stream
    qid = kid[:, query_offset:query_offset + S]
    ig = torch.arange(S).view(S, 1) + query_offset
    j = torch.arange(Skv).view(1, Skv)
    causal = j <= ig
    win = torch.ones_like(causal) if window == 0 else (ig - j) < window
    m = (valid.bool().view(B, S, 1) & key_valid.bool().view(B, 1, Skv)
         & (qid.view(B, S, 1) == kid.view(B, 1, Skv)) & (qid.view(B, S, 1) >= 0)
         & causal.view(1, S, Skv) & win.view(1, S, Skv))
    return m.view(B, 1, S, Skv).expand(B, heads_q, S, Skv)


def bias_matrix(profiles: torch.Tensor, *, seq_k: int, query_offset: int = 0) -> torch.Tensor:
    """[B,Hq,S,Skv] relative bias profiles[b,h,i,i_g-j] for 0 <= i_g-j < R, else 0 (differentiable)."""
    B, Hq, S, R = profiles.shape
    ig = torch.arange(S).view(S, 1) + query_offset
    j = torch.arange(seq_k).view(1, seq_k)
    d = ig - j
    inside = (d >= 0) & (d < R)
    idx = d.clamp(0, max(R - 1, 0)).view(1, 1, S, seq_k).expand(B, Hq, S, seq_k)
    if R == 0:
        return torch.zeros(B, Hq, S, seq_k, dtype=profiles.dtype)
    g = torch.gather(profiles, 3, idx)
    return torch.where(inside.view(1, 1, S, seq_k), g, torch.zeros((), dtype=profiles.dtype))


def logits(q, k, profiles, mask, *, query_offset=0):
    """[B,Hq,S,Skv] logits scale*q.k + bias, -inf where not allowed."""
    B, S, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kk = k.repeat_interleave(G, dim=2)              # [B,Skv,Hq,D]
    s = torch.einsum("bihd,bjhd->bhij", q, kk) * (D ** -0.5)
    z = s + bias_matrix(profiles, seq_k=Skv, query_offset=query_offset)
    return torch.where(mask, z, torch.full((), float("-inf"), dtype=z.dtype))


def forward(q, k, v, profiles, sink, mask, *, query_offset=0):
    """out [B,S,Hq,D], lse [B,S,Hq] through torch.logsumexp and softmax with a sink column."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    z = logits(q, k, profiles, mask, query_offset=query_offset)
    zs = torch.cat([z, sink.permute(0, 2, 1).unsqueeze(-1)], dim=-1)   # sink as an extra column
    lse = torch.logsumexp(zs, dim=-1)                                  # [B,Hq,S]
    p = torch.exp(zs - lse.unsqueeze(-1))[..., :-1]
    vv = v.repeat_interleave(G, dim=2)
    out = torch.einsum("bhij,bjhd->bihd", p, vv)
    return out, lse.permute(0, 2, 1)


def sdpa_forward(q, k, v, profiles, sink, mask, *, query_offset=0):
    """out through torch.nn.functional.scaled_dot_product_attention with an additive mask.

    The sink enters as one extra key whose key and value rows are zero and whose
    additive mask entry is the sink logit.
    """
    import torch.nn.functional as F
    B, S, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kk = k.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)            # [B,Hq,Skv,D]
    vv = v.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    qq = q.permute(0, 2, 1, 3)
    add = bias_matrix(profiles, seq_k=Skv, query_offset=query_offset)
    add = torch.where(mask, add, torch.full((), float("-inf"), dtype=add.dtype))
    add = torch.cat([add, sink.permute(0, 2, 1).unsqueeze(-1)], dim=-1)
    zk = torch.zeros(B, Hq, 1, D, dtype=q.dtype)
    out = F.scaled_dot_product_attention(qq, torch.cat([kk, zk], 2), torch.cat([vv, zk], 2),
                                         attn_mask=add, scale=D ** -0.5)
    return out.permute(0, 2, 1, 3)
