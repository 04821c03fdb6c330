"""FP64 CPU oracle for the generic FlexAttention variant.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers; the product path never imports it.

Semantics follow the NeMo AutoModel API page for
``nemo_automodel.components.attention.flex_attention.FlexAttention``:
``forward(q, k, v, scale, sink_weights, sliding_window, enable_gqa)`` with q
``[B, Hq, S, D]`` and k / v ``[B, Hkv, S, D]``, the ``attn_mask_type`` values
``"causal"`` and ``"block_causal"`` (blocks delimited by an EOS token),
``fixed_block_size`` and the sliding-window mask mod. The page states the
masks in words; this module writes each rule out as a boolean predicate on
(query index, key index) and evaluates attention densely, one (batch, head)
at a time, in float64 with numpy.

Readings where the page leaves a point open (the CUDA path encodes the same):

* F1 block_causal: a document ends with its EOS token (the EOS belongs to
  the document it closes); the token after an EOS starts a new document.
  Attention is causal inside a document and never crosses one.
* F2 fixed_block_size F > 0: each row of tokens is cut into blocks
  [kF, (k + 1)F) (the last one may be shorter); a query sees only keys of its
  own block. The rule is combined (AND) with the mask type.
* F3 sliding_window W > 0: a query sees the W most recent tokens including
  itself (i - j < W), as the forward describes the parameter (a count of
  causal tokens per query); the mask mod's inclusive bound q_idx - kv_idx <=
  window is the same rule with W + 1. W = 0: the full causal history.
* F4 sink_weights [Hq]: one logit per query head, acting as a virtual key
  with a zero value row in every row's softmax denominator; None = no sink.
* F5 scale: the page applies ``scale`` when sink_weights is not set; with
  sink weights the scale is head_dim^-0.5. None means head_dim^-0.5.
* F6 lse: log of the full denominator (sink included), [B, Hq, S].
* enable_gqa False requires Hq == Hkv; with it, query head h reads KV head
  h // (Hq / Hkv).
"""
from __future__ import annotations

from typing import Optional

import numpy as np

MASK_TYPES = ("causal", "block_causal")


def effective_scale(head_dim: int, scale: Optional[float], sink_weights) -> float:
    """F5: the scale that multiplies q.k."""
    if sink_weights is None and scale is not None:
        return float(scale)
    return float(head_dim) ** -0.5


def document_ids(tokens_row: np.ndarray, eos_id: int) -> np.ndarray:
    """F1: document index of every token = number of EOS tokens strictly before it."""
    is_eos = (np.asarray(tokens_row) == eos_id).astype(np.int64)
    before = np.concatenate([[0], np.cumsum(is_eos)[:-1]])
    return before


def allowed(S: int, mask_type: str, tokens_row=None, eos_id: Optional[int] = None,
            fixed_block_size: int = 0, sliding_window: int = 0) -> np.ndarray:
    """bool [S, S]: allowed[i, j] for query i and key j of one batch row."""
    if mask_type not in MASK_TYPES:
        raise ValueError(f"mask_type must be one of {MASK_TYPES}")
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    m = j <= i                                   # causal
    if mask_type == "block_causal":
        if tokens_row is None or eos_id is None:
            raise ValueError("block_causal needs tokens and eos_id")
        doc = document_ids(tokens_row, eos_id)
        m &= doc[:, None] == doc[None, :]
    if fixed_block_size > 0:
        m &= (i // fixed_block_size) == (j // fixed_block_size)
    if sliding_window > 0:
        m &= (i - j) < sliding_window
    return m


def _check(q, k, v, enable_gqa):
    B, Hq, S, D = q.shape
    if k.shape[0] != B or k.shape[2] != S or k.shape[3] != D or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, S, D] with the q's B, S and D")
    Hkv = k.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    if Hq != Hkv and not enable_gqa:
        raise ValueError("Hq != Hkv needs enable_gqa")
    return B, Hq, Hkv, S, D


def _probabilities(q_bh, k_bg, mask, scale, sigma):
    """Scores, full-denominator lse (sink included) and probabilities of one (b, h)."""
    s = scale * (q_bh @ k_bg.T)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1)
    if sigma is not None:
        m = np.maximum(m, sigma)
    z = np.exp(s - m[:, None]).sum(axis=1)
    if sigma is not None:
        z = z + np.exp(sigma - m)
    lse = m + np.log(z)
    p = np.exp(s - lse[:, None])
    return s, lse, p


def forward(q, k, v, sink_weights=None, tokens=None, *, mask_type: str = "causal", eos_id: Optional[int] = None,
            fixed_block_size: int = 0, sliding_window: int = 0, scale: Optional[float] = None,
            enable_gqa: bool = False):
    """out [B, Hq, S, D] and lse [B, Hq, S], float64."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, Hq, Hkv, S, D = _check(q, k, v, enable_gqa)
    sc = effective_scale(D, scale, sink_weights)
    sw = None if sink_weights is None else np.asarray(sink_weights, dtype=np.float64)
    out = np.zeros(q.shape)
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        mask = allowed(S, mask_type, None if tokens is None else tokens[b], eos_id, fixed_block_size,
                       sliding_window)
        for h in range(Hq):
            g = h // (Hq // Hkv)
            _, lse[b, h], p = _probabilities(q[b, h], k[b, g], mask, sc, None if sw is None else sw[h])
            out[b, h] = p @ v[b, g]
    return out, lse


def backward(q, k, v, sink_weights=None, tokens=None, *, dout, mask_type: str = "causal",
             eos_id: Optional[int] = None, fixed_block_size: int = 0, sliding_window: int = 0,
             scale: Optional[float] = None, enable_gqa: bool = False):
    """Gradients of sum(dout * out): dict dq, dk, dv (float64, layouts of q / k / v) and
    dsink_weights [Hq] (None without sink weights).

    Per (b, h): P from the recomputed scores, Dv_i = sum_d dO.O, dP = dO V^T,
    dS = P (dP - Dv), dQ = scale dS K, dK += scale dS^T Q, dV += P^T dO, and for the
    sink logit d sigma_h += sum_i -p_sink,i Dv_i with p_sink,i = exp(sigma_h - lse_i).
    """
    q, k, v, dout = (np.asarray(t, dtype=np.float64) for t in (q, k, v, dout))
    B, Hq, Hkv, S, D = _check(q, k, v, enable_gqa)
    sc = effective_scale(D, scale, sink_weights)
    sw = None if sink_weights is None else np.asarray(sink_weights, dtype=np.float64)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    dsw = None if sw is None else np.zeros(Hq)
    for b in range(B):
        mask = allowed(S, mask_type, None if tokens is None else tokens[b], eos_id, fixed_block_size,
                       sliding_window)
        for h in range(Hq):
            g = h // (Hq // Hkv)
            sigma = None if sw is None else sw[h]
            _, lse, p = _probabilities(q[b, h], k[b, g], mask, sc, sigma)
            o = p @ v[b, g]
            dvec = (dout[b, h] * o).sum(axis=1)
            dp = dout[b, h] @ v[b, g].T
            ds = p * (dp - dvec[:, None])
            dq[b, h] = sc * (ds @ k[b, g])
            dk[b, g] += sc * (ds.T @ q[b, h])
            dv[b, g] += p.T @ dout[b, h]
            if dsw is not None:
                dsw[h] += float((-np.exp(sigma - lse) * dvec).sum())
    return dict(dq=dq, dk=dk, dv=dv, dsink_weights=dsw)
