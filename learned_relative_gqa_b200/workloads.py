"""Named workloads and the seeded synthetic input generator.

This module holds shapes, distributions and random draws only -- none of the
attention arithmetic -- so that the CUDA path and the FP64 oracle can be fed
identical inputs without sharing any code of the method.

Workloads (shapes and value distributions of the Inkling2 attention layers
described on the NeMo AutoModel pages for ``Inkling2FlexAttention`` /
``Inkling2Attention``):

====================  ==============================================================
``pr1_ref``           B1 S128 Hq4 Hkv2 D64, full causal, R=64, one document, all valid
``local``             B2 S2048 Hq16 Hkv4 D128, window 512, R=512, trailing padding
                      of U{0..127} tokens per row
``packed``            B4 S4096 Hq32 Hkv8 D128, causal within documents of
                      length U{256..2048}, R=1024
``long``              B1 S32768 Hq32 Hkv8 D128, full causal, R=4096, one document
``train``             B2 S8192 Hq32 Hkv4 D128, window 1024, R=1024, documents of
                      length U{512..4096}, forward + backward with dO ~ N(0,1) FP32
====================  ==============================================================

Recipe (identical for every workload, seed = 1000 + workload index):

* float draws on a ``torch.Generator`` of the target device seeded with the
  seed, in this order: q, k, v ~ N(0,1) rounded to BF16 (round-to-nearest-even,
  ``Tensor.to(torch.bfloat16)``); profiles ~ N(0, 0.5^2) rounded to BF16 (0.5 is
  the standard deviation); sink ~ N(0,1) FP32; dO ~ N(0,1) FP32 (backward only);
* integer draws (padding lengths, then document lengths) on a CPU generator
  seeded with the same seed, so the mask structure is the same on every device;
* padding p ~ U{lo..hi} per batch row: the last p tokens are invalid and get
  position 0; documents: lengths ~ U{lo..hi} drawn until they cover the row, the
  last one truncated; positions restart at 0 in each document.
* key tensors equal the query-side ones (key_valid = valid, key_positions =
  positions, query_offset = 0) except in the context-parallel test shapes, where
  the query side is a slice [query_offset, query_offset + S) of the global key
  stream.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seq: int
    heads_q: int
    heads_kv: int
    head_dim: int
    window: int            # 0 = full causal
    rel_extent: int
    docs: Optional[Tuple[int, int]] = None     # document length range (inclusive)
    pad: Optional[Tuple[int, int]] = None      # trailing padding range (inclusive)
    backward: bool = False
    seq_k: Optional[int] = None                # global key length (context-parallel shapes)
    query_offset: int = 0

    @property
    def skv(self) -> int:
        return self.seq if self.seq_k is None else self.seq_k


WORKLOADS = [
    Workload("pr1_ref", 1, 128, 4, 2, 64, 0, 64),
    Workload("local", 2, 2048, 16, 4, 128, 512, 512, pad=(0, 127)),
    Workload("packed", 4, 4096, 32, 8, 128, 0, 1024, docs=(256, 2048)),
    Workload("long", 1, 32768, 32, 8, 128, 0, 4096),
    Workload("train", 2, 8192, 32, 4, 128, 1024, 1024, docs=(512, 4096), backward=True),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def seed_of(w: Workload) -> int:
    for idx, x in enumerate(WORKLOADS):
        if x.name == w.name:
            return 1000 + idx
    return 2000 + (zlib.crc32(repr(w).encode()) & 0xFFFF)


def _structure(w: Workload, seed: int):
    """valid / positions for the global key stream (CPU, int draws only)."""
    g = torch.Generator("cpu")
    g.manual_seed(seed)
    B, T = w.batch, w.skv
    valid = torch.ones(B, T, dtype=torch.bool)
    positions = torch.zeros(B, T, dtype=torch.int32)
    pads = [0] * B
    if w.pad is not None:
        lo, hi = w.pad
        pads = [int(torch.randint(lo, hi + 1, (1,), generator=g)) for _ in range(B)]
    for b in range(B):
        n_real = T - pads[b]
        if w.docs is None:
            lengths = [n_real]
        else:
            lo, hi = w.docs
            lengths, total = [], 0
            while total < n_real:
                L = int(torch.randint(lo, hi + 1, (1,), generator=g))
                L = min(L, n_real - total)
                lengths.append(L)
                total += L
        c = 0
        for L in lengths:
            positions[b, c:c + L] = torch.arange(L, dtype=torch.int32)
            c += L
        valid[b, n_real:] = False
        positions[b, n_real:] = 0
    return valid, positions


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None, with_dout: Optional[bool] = None):
    """Draw the synthetic inputs for workload ``w`` on ``device``.

    Returns a dict with q, k, v, profiles (BF16), sink (FP32), valid, key_valid
    (bool), positions, key_positions (int32), dout (FP32, backward workloads) and the
    scalar fields window, rel_extent, query_offset.
    """
    seed = seed_of(w) if seed is None else seed
    with_dout = w.backward if with_dout is None else with_dout
    dev = torch.device(device)
    g = torch.Generator(dev)
    g.manual_seed(seed)
    B, S, Hq, Hkv, D, R, T = w.batch, w.seq, w.heads_q, w.heads_kv, w.head_dim, w.rel_extent, w.skv

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    q = randn(B, S, Hq, D).to(torch.bfloat16)
    k = randn(B, T, Hkv, D).to(torch.bfloat16)
    v = randn(B, T, Hkv, D).to(torch.bfloat16)
    # profiles are drawn row-block by row-block to bound the FP32 staging buffer
    profiles = torch.empty(B, Hq, S, R, dtype=torch.bfloat16, device=dev)
    for b in range(B):
        for h in range(Hq):
            profiles[b, h] = (randn(S, R) * 0.5).to(torch.bfloat16)
    sink = randn(B, S, Hq)
    dout = randn(B, S, Hq, D) if with_dout else None

    kvalid, kpos = _structure(w, seed)
    off = w.query_offset
    valid = kvalid[:, off:off + S].contiguous()
    positions = kpos[:, off:off + S].contiguous()
    return dict(
        q=q, k=k, v=v, profiles=profiles, sink=sink, dout=dout,
        valid=valid.to(dev), key_valid=kvalid.to(dev),
        positions=positions.to(dev), key_positions=kpos.to(dev),
        window=w.window, rel_extent=R, query_offset=off,
    )


def allowed_counts(w: Workload, inputs) -> int:
    """Number E of allowed (query row, key, head) triples, for FLOP accounting.

    Counted from the mask structure on the host: a valid row i (global column
    i_g) attends the valid keys j <= i_g of its own document inside the window.
    """
    valid = inputs["valid"].cpu()
    kvalid = inputs["key_valid"].cpu()
    pos = inputs["positions"].cpu().to(torch.int64)
    kpos = inputs["key_positions"].cpu().to(torch.int64)
    off = inputs["query_offset"]
    W = inputs["window"]
    B, S = valid.shape
    total = 0
    ig = torch.arange(S, dtype=torch.int64) + off
    for b in range(B):
        kv = kvalid[b]
        idx = torch.nonzero(kv).flatten()
        if idx.numel() == 0:
            continue
        kfirst, klast = int(idx[0]), int(idx[-1])
        lo = torch.maximum(ig - pos[b], torch.full_like(ig, kfirst))
        if W > 0:
            lo = torch.maximum(lo, ig - W + 1)
        hi = torch.minimum(ig, torch.full_like(ig, klast))
        cnt = (hi - lo + 1).clamp(min=0) * valid[b].to(torch.int64)
        total += int(cnt.sum())
    del kpos
    return total * w.heads_q


# --------------------------------------------------------------------------
# generic FlexAttention variant (NeMo AutoModel ``FlexAttention`` module page):
# [B, H, S, D] layout, per-head sink weights, EOS-delimited documents
# --------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class FlexWorkload:
    name: str
    batch: int
    seq: int
    heads_q: int
    heads_kv: int
    head_dim: int
    mask_type: str = "causal"                  # "causal" or "block_causal"
    docs: Optional[Tuple[int, int]] = None     # document length range (block_causal), EOS closes each
    fixed_block_size: int = 0
    sliding_window: int = 0
    sink: bool = True                          # draw sink_weights [Hq]
    scale: Optional[float] = None
    eos_id: int = 2
    vocab: int = 32000


FLEX_WORKLOADS = [
    # the packed-documents shape with EOS-delimited documents, per-head sinks
    FlexWorkload("flex_packed", 4, 4096, 32, 8, 128, "block_causal", docs=(256, 2048)),
]
FLEX_BY_NAME = {w.name: w for w in FLEX_WORKLOADS}


def flex_seed_of(w: FlexWorkload) -> int:
    for idx, x in enumerate(FLEX_WORKLOADS):
        if x.name == w.name:
            return 3000 + idx
    return 4000 + (zlib.crc32(repr(w).encode()) & 0xFFFF)


def make_flex_inputs(w: FlexWorkload, device="cpu", seed: Optional[int] = None, with_dout: bool = True):
    """q [B,Hq,S,D], k / v [B,Hkv,S,D] ~ N(0,1) rounded to BF16, sink_weights [Hq] ~ N(0,1)
    FP32 (or None), tokens [B,S] int64 and dout [B,Hq,S,D] ~ N(0,1) rounded to BF16.

    Float draws on a generator of the target device (q, k, v, sink_weights, dout in that
    order); tokens on a CPU generator with the same seed: ids uniform in [0, vocab)
    without the EOS id, then document lengths ~ U{lo..hi} drawn until they cover the
    row, the last one truncated, and the EOS id placed on the last token of every
    complete document.
    """
    seed = flex_seed_of(w) if seed is None else seed
    dev = torch.device(device)
    g = torch.Generator(dev)
    g.manual_seed(seed)
    B, S, Hq, Hkv, D = w.batch, w.seq, w.heads_q, w.heads_kv, w.head_dim

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    q = randn(B, Hq, S, D).to(torch.bfloat16)
    k = randn(B, Hkv, S, D).to(torch.bfloat16)
    v = randn(B, Hkv, S, D).to(torch.bfloat16)
    sink = randn(Hq) if w.sink else None
    dout = randn(B, Hq, S, D).to(torch.bfloat16) if with_dout else None

    gc = torch.Generator("cpu")
    gc.manual_seed(seed)
    tokens = torch.randint(0, w.vocab - 1, (B, S), generator=gc, dtype=torch.int64)
    tokens = tokens + (tokens >= w.eos_id).to(torch.int64)        # never the EOS id
    if w.docs is not None:
        lo, hi = w.docs
        for b in range(B):
            c = 0
            while c < S:
                L = int(torch.randint(lo, hi + 1, (1,), generator=gc))
                if c + L <= S:
                    tokens[b, c + L - 1] = w.eos_id
                c += L
    return dict(q=q, k=k, v=v, sink_weights=sink, tokens=tokens.to(dev), dout=dout,
                mask_type=w.mask_type, eos_id=w.eos_id, fixed_block_size=w.fixed_block_size,
                sliding_window=w.sliding_window, scale=w.scale, enable_gqa=Hq != Hkv)


def flex_allowed_counts(w: FlexWorkload, inputs) -> int:
    """Number E of allowed (query, key, head) triples of a generic-variant input, for FLOP
    accounting: per batch row, the blocks (documents closed by EOS, cut further at
    multiples of fixed_block_size) each contribute the causal pairs inside them, capped
    by the sliding window."""
    tokens = inputs["tokens"].cpu()
    B, S = tokens.shape
    total = 0
    for b in range(B):
        starts = [0]
        for c in range(1, S):
            if (w.mask_type == "block_causal" and int(tokens[b, c - 1]) == w.eos_id) or \
                    (w.fixed_block_size > 0 and c % w.fixed_block_size == 0):
                starts.append(c)
        starts.append(S)
        for a, e in zip(starts[:-1], starts[1:]):
            L = e - a
            if w.sliding_window > 0 and w.sliding_window < L:
                W = w.sliding_window
                total += W * (W + 1) // 2 + (L - W) * W
            else:
                total += L * (L + 1) // 2
    return total * w.heads_q

