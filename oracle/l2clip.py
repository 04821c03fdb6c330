"""FP64 CPU oracle for L2Clip, the per-head clipping applied to q and k ahead of
the attention.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers; the product path never imports it.

Follows the NeMo AutoModel API page for
``nemo_automodel.components.models.inkling2.layers``: ``L2Clip(heads, width,
threshold, learned_scale)`` clips each head's vector by its L2 norm, with
optional learned per-channel scales in front, and ``L2Clip.forward(x [batch,
sequence, heads, head_dim], tau [batch, sequence] | None)`` applies tau as a
length scaling after the clip and returns x's dtype.

The page names the operation but prints no formula; this module takes the
plainest reading (the CUDA path encodes the same):

* L1 learned scales: a weight ``scale [heads, width]`` multiplies x channel by
  channel before the clipping; without learned_scale there is none.
* L2 clipping: z = x * scale per (batch, token, head) vector;
  y = z * min(1, threshold / ||z||_2). Vectors inside the ball are unchanged,
  longer ones are shortened to length ``threshold`` along their direction.
* L3 length scaling: y <- y * tau[b, s] after the clipping.
* L4 arithmetic in FP64 here (FP32 on the GPU), the result rounded to x's dtype
  by the caller.

Gradient (of sum(dy * y)), at ||z|| > threshold with c = threshold / ||z||:
dz = tau * c * (dy - ((z . dy) / ||z||^2) z); at ||z|| <= threshold: dz = tau * dy
(the ball's boundary takes the inside branch). dx = dz * scale,
dscale[h, :] = sum over (b, s) of dz * x, dtau[b, s] = sum over (h, d) of dy * z * c.

The clipping rule is a reading of the page, not a formula it prints: the pins
tie this module to the mathematics of that rule (closed forms, invariants,
autograd, finite differences), not to a value the page gives ("parity
unpinned" against the page itself).
"""
from __future__ import annotations

from typing import Optional

import numpy as np


def forward(x, scale: Optional[np.ndarray], tau: Optional[np.ndarray], threshold: float) -> np.ndarray:
    """y [B, S, H, D] float64."""
    x = np.asarray(x, dtype=np.float64)
    z = x * (1.0 if scale is None else np.asarray(scale, dtype=np.float64)[None, None])
    n = np.sqrt((z * z).sum(axis=-1, keepdims=True))
    c = np.where(n > threshold, threshold / np.where(n > 0, n, 1.0), 1.0)
    y = z * c
    if tau is not None:
        y = y * np.asarray(tau, dtype=np.float64)[:, :, None, None]
    return y


def backward(x, scale: Optional[np.ndarray], tau: Optional[np.ndarray], threshold: float, dy):
    """dict dx [B,S,H,D], dscale [H,D] (None without scale), dtau [B,S] (None without tau)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    sc = None if scale is None else np.asarray(scale, dtype=np.float64)
    z = x * (1.0 if sc is None else sc[None, None])
    n = np.sqrt((z * z).sum(axis=-1, keepdims=True))
    clipped = n > threshold
    c = np.where(clipped, threshold / np.where(n > 0, n, 1.0), 1.0)
    t = 1.0 if tau is None else np.asarray(tau, dtype=np.float64)[:, :, None, None]
    zdy = (z * dy).sum(axis=-1, keepdims=True)
    n2 = np.where(clipped, n * n, 1.0)
    dz = np.where(clipped, t * c * (dy - (zdy / n2) * z), t * dy)
    dx = dz if sc is None else dz * sc[None, None]
    dscale = None if sc is None else (dz * x).sum(axis=(0, 1))
    dtau = None if tau is None else (dy * z * c).sum(axis=(2, 3))
    return dict(dx=dx, dscale=dscale, dtau=dtau)
