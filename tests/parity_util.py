"""Helpers for the GPU-vs-oracle parity tests.

Tolerances (stated by the task for this method): outputs max |err| <= 1e-2 and
mean |err| <= 1e-3; log-sum-exp within 1e-3 (absolute); gradients within 2e-2
relative, read per gradient tensor as max |g - g_ref| <= 2e-2 * max |g_ref|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from learned_relative_gqa_b200 import binding
from learned_relative_gqa_b200 import workloads as W

OUT_MAX, OUT_MEAN, LSE_TOL, GRAD_REL = 1e-2, 1e-3, 1e-3, 2e-2


def to_host(x: dict) -> dict:
    """float64 numpy copies of the device inputs (BF16 decoded by the oracle's own routine)."""
    h = {}
    for n in ("q", "k", "v", "profiles"):
        h[n] = oracle.decode_bf16(x[n].cpu().view(torch.int16).numpy())
    h["sink"] = x["sink"].cpu().double().numpy()
    for n in ("valid", "key_valid"):
        h[n] = x[n].cpu().numpy().astype(np.uint8)
    for n in ("positions", "key_positions"):
        h[n] = x[n].cpu().numpy().astype(np.int32)
    if x.get("dout") is not None:
        h["dout"] = x["dout"].cpu().double().numpy()
    h["window"], h["query_offset"] = x["window"], x["query_offset"]
    return h


def gpu_forward(x: dict):
    return binding.forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                           x["positions"], x["key_positions"], window=x["window"], query_offset=x["query_offset"])


def gpu_backward(x: dict, out, lse, dlse=None):
    return binding.backward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                            x["positions"], x["key_positions"], out, lse, x["dout"], dlse,
                            window=x["window"], query_offset=x["query_offset"])


def oracle_forward(h: dict, rows=None):
    return oracle.forward(h["q"], h["k"], h["v"], h["profiles"], h["sink"], h["valid"], h["key_valid"],
                          h["positions"], h["key_positions"], window=h["window"], query_offset=h["query_offset"],
                          rows=rows)


def oracle_backward(h: dict, dlse=None):
    return oracle.backward(h["q"], h["k"], h["v"], h["profiles"], h["sink"], h["valid"], h["key_valid"],
                           h["positions"], h["key_positions"], dout=h["dout"], dlse=dlse, window=h["window"],
                           query_offset=h["query_offset"])


def assert_out_close(out_gpu, out_ref, what="out"):
    o = np.asarray(out_gpu, dtype=np.float64)
    err = np.abs(o - out_ref)
    assert np.all(np.isfinite(o)), f"{what}: non-finite values"
    assert err.max() <= OUT_MAX, f"{what}: max abs err {err.max():.3e} > {OUT_MAX}"
    assert err.mean() <= OUT_MEAN, f"{what}: mean abs err {err.mean():.3e} > {OUT_MEAN}"
    return float(err.max()), float(err.mean())


def assert_lse_close(lse_gpu, lse_ref, what="lse"):
    a = np.asarray(lse_gpu, dtype=np.float64)
    both_inf = np.isinf(a) & np.isinf(lse_ref) & (np.sign(a) == np.sign(lse_ref))
    err = np.where(both_inf, 0.0, np.abs(a - lse_ref))
    assert err.max() <= LSE_TOL, f"{what}: max abs err {err.max():.3e} > {LSE_TOL}"
    return float(err.max())


def assert_grad_close(g_gpu, g_ref, what):
    g = np.asarray(g_gpu, dtype=np.float64)
    assert g.shape == np.shape(g_ref), f"{what}: shape {g.shape} vs {np.shape(g_ref)}"
    if g.size == 0:
        return 0.0
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    scale = max(float(np.abs(g_ref).max()), 1e-30)
    err = float(np.abs(g - g_ref).max())
    assert err <= GRAD_REL * scale, f"{what}: max abs err {err:.3e} > {GRAD_REL} * {scale:.3e}"
    return err / scale


def sample_rows(x: dict, n: int, seed: int = 0) -> np.ndarray:
    """Flattened (b*S+i)*Hq+h row ids: document starts and ends, the last rows, and random rows."""
    B, S, Hq = x["q"].shape[:3]
    pos = x["positions"].cpu().numpy()
    valid = x["valid"].cpu().numpy().astype(bool)
    rng = np.random.default_rng(seed)
    picks = set()
    for b in range(B):
        starts = np.nonzero((pos[b] == 0) & valid[b])[0]
        for s in starts[: max(1, n // (8 * B))]:
            for i in (s, min(S - 1, s + 1), max(0, s - 1)):
                picks.add((b, int(i)))
        for i in (S - 1, S - 2, 0, S // 2):
            picks.add((b, max(0, i)))
    while len(picks) < n // 2:
        picks.add((int(rng.integers(B)), int(rng.integers(S))))
    rows = []
    for (b, i) in sorted(picks):
        for h in rng.choice(Hq, size=min(2, Hq), replace=False):
            rows.append((b * S + i) * Hq + int(h))
    return np.array(sorted(set(rows)), dtype=np.int64)


def custom(name, B, S, Hq, Hkv, D, window, R, docs=None, pad=None, seq_k=None, query_offset=0, backward=True):
    return W.Workload(name, B, S, Hq, Hkv, D, window, R, docs=docs, pad=pad, backward=backward, seq_k=seq_k,
                      query_offset=query_offset)
