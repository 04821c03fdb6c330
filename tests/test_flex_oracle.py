"""Pins for the FP64 oracle of the generic FlexAttention variant (CPU only).

Each check compares the oracle with something other than itself: values worked
out by hand, torch's scaled_dot_product_attention on masks built here by walking
the tokens one by one, closed forms of the sink, special cases whose result is
known, torch autograd of a dense formulation, finite differences of the
oracle's own forward, and the (separately pinned) learned-relative oracle with
no profiles.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import flex
from learned_relative_gqa_b200 import workloads as W


def inputs(B=2, S=37, Hq=4, Hkv=2, D=8, mask_type="block_causal", docs=(3, 11), fbs=0, win=0, sink=True,
           scale=None, seed=None):
    w = W.FlexWorkload("pin", B, S, Hq, Hkv, D, mask_type, docs=docs, fixed_block_size=fbs, sliding_window=win,
                       sink=sink, scale=scale)
    x = W.make_flex_inputs(w, "cpu", seed=seed)
    for n in ("q", "k", "v", "dout"):
        x[n] = x[n].double()
    if x["sink_weights"] is not None:
        x["sink_weights"] = x["sink_weights"].double()
    return x


def fwd(x, **over):
    kw = dict(mask_type=x["mask_type"], eos_id=x["eos_id"], fixed_block_size=x["fixed_block_size"],
              sliding_window=x["sliding_window"], scale=x["scale"], enable_gqa=x["enable_gqa"])
    kw.update(over)
    sw = x["sink_weights"]
    return flex.forward(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), None if sw is None else sw.numpy(),
                        x["tokens"].numpy(), **kw)


def bwd(x, **over):
    kw = dict(mask_type=x["mask_type"], eos_id=x["eos_id"], fixed_block_size=x["fixed_block_size"],
              sliding_window=x["sliding_window"], scale=x["scale"], enable_gqa=x["enable_gqa"])
    kw.update(over)
    sw = x["sink_weights"]
    return flex.backward(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), None if sw is None else sw.numpy(),
                         x["tokens"].numpy(), dout=x["dout"].numpy(), **kw)


def walked_mask(tokens_row, S, mask_type, eos_id, fbs, win):
    """allowed[i, j] by walking the sequence: a document counter that steps after each EOS."""
    doc = []
    d = 0
    for t in range(S):
        doc.append(d)
        if mask_type == "block_causal" and int(tokens_row[t]) == eos_id:
            d += 1
    m = torch.zeros(S, S, dtype=torch.bool)
    for i in range(S):
        for j in range(i + 1):
            ok = doc[i] == doc[j]
            if fbs > 0:
                ok = ok and (i // fbs == j // fbs)
            if win > 0:
                ok = ok and (i - j <= win - 1)
            m[i, j] = ok
    return m


# --------------------------------------------------------------------------
# 1. values worked out by hand
# --------------------------------------------------------------------------
def test_tiny_block_causal_by_hand():
    # B=1, H=1, D=1 (scale 1), tokens [5, EOS, 7]: documents {0, 1} and {2}
    q = np.array([1.0, 2.0, 3.0]).reshape(1, 1, 3, 1)
    k = np.array([1.0, 1.0, 2.0]).reshape(1, 1, 3, 1)
    v = np.array([1.0, 3.0, 5.0]).reshape(1, 1, 3, 1)
    tokens = np.array([[5, 2, 7]])
    out, lse = flex.forward(q, k, v, None, tokens, mask_type="block_causal", eos_id=2)
    # row 0: key 0 alone; row 1: keys 0, 1 with equal scores 2; row 2: key 2 alone (score 6)
    np.testing.assert_allclose(out.reshape(-1), [1.0, 2.0, 5.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse.reshape(-1), [1.0, 2.0 + math.log(2.0), 6.0], rtol=0, atol=1e-15)
    # with a sink logit 0: row 0 has weights e^1 (key) and 1 (sink)
    out_s, lse_s = flex.forward(q, k, v, np.array([0.0]), tokens, mask_type="block_causal", eos_id=2)
    np.testing.assert_allclose(out_s[0, 0, 0, 0], math.e / (1.0 + math.e), rtol=1e-15)
    np.testing.assert_allclose(lse_s[0, 0, 0], math.log(1.0 + math.e), rtol=1e-15)
    # plain causal: row 2 sees all three keys, scores 3, 3, 6
    out_c, _ = flex.forward(q, k, v, None, None, mask_type="causal")
    e3, e6 = math.exp(3.0), math.exp(6.0)
    np.testing.assert_allclose(out_c[0, 0, 2, 0], (e3 * 1 + e3 * 3 + e6 * 5) / (2 * e3 + e6), rtol=1e-14)


# --------------------------------------------------------------------------
# 2. library routine on masks built independently
# --------------------------------------------------------------------------
@pytest.mark.parametrize("scale", [None, 0.3])
def test_causal_without_sinks_is_sdpa(scale):
    x = inputs(mask_type="causal", docs=None, sink=False, scale=scale)
    out, lse = fwd(x)
    ref = F.scaled_dot_product_attention(x["q"], x["k"], x["v"], is_causal=True, scale=scale, enable_gqa=True)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("fbs,win", [(0, 0), (8, 0), (0, 5), (6, 4)])
def test_block_causal_fixed_blocks_and_window_are_sdpa_with_walked_masks(fbs, win):
    x = inputs(fbs=fbs, win=win, sink=False)
    out, _ = fwd(x)
    B, Hq, S, D = x["q"].shape
    for b in range(B):
        m = walked_mask(x["tokens"][b], S, "block_causal", x["eos_id"], fbs, win)
        ref = F.scaled_dot_product_attention(x["q"][b:b + 1], x["k"][b:b + 1], x["v"][b:b + 1], attn_mask=m,
                                             enable_gqa=True)
        np.testing.assert_allclose(out[b:b + 1], ref.numpy(), rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# 3. closed forms and special cases
# --------------------------------------------------------------------------
def test_sink_is_a_closed_form_of_the_sinkless_result():
    x = inputs()
    out_s, lse_s = fwd(x)
    out_n, lse_n = fwd({**x, "sink_weights": None})
    sigma = x["sink_weights"].numpy()[None, :, None]
    p_sink = 1.0 / (1.0 + np.exp(lse_n - sigma))
    np.testing.assert_allclose(lse_s, np.logaddexp(lse_n, sigma), rtol=1e-13)
    np.testing.assert_allclose(out_s, out_n * (1.0 - p_sink)[..., None], rtol=1e-11, atol=1e-13)


def test_fixed_block_of_one_and_window_of_one_return_v():
    x = inputs(sink=False)
    G = x["q"].shape[1] // x["k"].shape[1]
    v_rep = np.repeat(x["v"].numpy(), G, axis=1)
    k_rep = np.repeat(x["k"].numpy(), G, axis=1)
    diag = (x["q"].numpy() * k_rep).sum(-1) * x["q"].shape[-1] ** -0.5
    for kw in (dict(fixed_block_size=1), dict(sliding_window=1)):
        out, lse = fwd(x, **kw)
        np.testing.assert_allclose(out, v_rep, rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse, diag, rtol=1e-14, atol=1e-14)


def test_window_and_block_at_least_the_sequence_change_nothing():
    x = inputs()
    out0, lse0 = fwd(x)
    S = x["q"].shape[2]
    for kw in (dict(sliding_window=S), dict(fixed_block_size=S)):
        out, lse = fwd(x, **kw)
        np.testing.assert_array_equal(out, out0)
        np.testing.assert_array_equal(lse, lse0)


def test_scale_is_not_applied_with_sink_weights():
    x = inputs()
    a = fwd(x, scale=0.3)
    b = fwd(x, scale=None)
    np.testing.assert_array_equal(a[0], b[0])
    xn = {**x, "sink_weights": None}
    c = fwd(xn, scale=0.3)
    d = fwd(xn, scale=None)
    assert np.abs(c[0] - d[0]).max() > 1e-3


def test_gqa_needs_enable_gqa():
    x = inputs()
    with pytest.raises(ValueError):
        fwd(x, enable_gqa=False)


def test_gqa_equals_mha_with_replicated_kv():
    x = inputs()
    G = x["q"].shape[1] // x["k"].shape[1]
    xr = {**x, "k": x["k"].repeat_interleave(G, 1), "v": x["v"].repeat_interleave(G, 1)}
    a = fwd(x)
    b = fwd(xr, enable_gqa=False)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-14, atol=1e-15)


def test_matches_the_learned_relative_oracle_without_profiles():
    """Documents from EOS tokens + fixed blocks, expressed as positions that restart at
    every block start, through the (separately pinned) C oracle with R = 0."""
    x = inputs(fbs=9, win=6)
    out, lse = fwd(x)
    B, Hq, S, D = x["q"].shape
    pos = np.zeros((B, S), np.int32)
    for b in range(B):
        start = 0
        for i in range(S):
            if i > 0 and (int(x["tokens"][b, i - 1]) == x["eos_id"] or i % 9 == 0):
                start = i
            pos[b, i] = i - start
    sink = np.broadcast_to(x["sink_weights"].numpy()[None, None, :], (B, S, Hq)).copy()
    o2, l2, _ = oracle.forward(x["q"].numpy().transpose(0, 2, 1, 3), x["k"].numpy().transpose(0, 2, 1, 3),
                               x["v"].numpy().transpose(0, 2, 1, 3), np.zeros((B, Hq, S, 0)), sink,
                               np.ones((B, S), np.uint8), positions=pos, window=6)
    np.testing.assert_allclose(out, o2.transpose(0, 2, 1, 3), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lse, l2.transpose(0, 2, 1), rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# 4. backward: autograd of a dense formulation, finite differences
# --------------------------------------------------------------------------
def dense_loss(q, k, v, sw, mask, scale, dout):
    G = q.shape[1] // k.shape[1]
    kk = k.repeat_interleave(G, 1)
    vv = v.repeat_interleave(G, 1)
    s = torch.einsum("bhid,bhjd->bhij", q, kk) * scale
    s = s.masked_fill(~mask[:, None], float("-inf"))
    col = sw.view(1, -1, 1, 1).expand(s.shape[0], s.shape[1], s.shape[2], 1)
    p = torch.softmax(torch.cat([s, col], dim=-1), dim=-1)[..., :-1]
    return (torch.einsum("bhij,bhjd->bhid", p, vv) * dout).sum()


@pytest.mark.parametrize("fbs,win", [(0, 0), (7, 5)])
def test_backward_matches_autograd(fbs, win):
    x = inputs(fbs=fbs, win=win)
    B, Hq, S, D = x["q"].shape
    mask = torch.stack([walked_mask(x["tokens"][b], S, "block_causal", x["eos_id"], fbs, win) for b in range(B)])
    leaves = {n: x[n].clone().requires_grad_(True) for n in ("q", "k", "v", "sink_weights")}
    dense_loss(leaves["q"], leaves["k"], leaves["v"], leaves["sink_weights"], mask, D ** -0.5, x["dout"]).backward()
    g = bwd(x)
    for n, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("sink_weights", "dsink_weights")):
        np.testing.assert_allclose(g[key], leaves[n].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=key)


def test_backward_finite_differences():
    x = inputs(B=1, S=11, Hq=2, Hkv=1, D=3, docs=(3, 6), fbs=5, win=4, seed=5)
    g = bwd(x)
    dout = x["dout"].numpy()

    def loss(xx):
        o, _ = fwd(xx)
        return float((o * dout).sum())

    h = 1e-6
    rng = np.random.default_rng(1)
    for n, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("sink_weights", "dsink_weights")):
        base = x[n]
        for t in rng.choice(base.numel(), size=min(10, base.numel()), replace=False):
            plus = {**x, n: base.clone()}
            minus = {**x, n: base.clone()}
            plus[n].view(-1)[t] += h
            minus[n].view(-1)[t] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            an = g[key].reshape(-1)[t]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (key, int(t), fd, an)


def test_generator_places_eos_at_document_ends():
    w = W.FlexWorkload("gen", 3, 300, 2, 1, 8, "block_causal", docs=(20, 60))
    x = W.make_flex_inputs(w)
    for b in range(3):
        ends = torch.nonzero(x["tokens"][b] == w.eos_id).flatten()
        gaps = torch.diff(torch.cat([torch.tensor([-1]), ends]))
        assert ends.numel() >= 4 and int(gaps.min()) >= 20 and int(gaps.max()) <= 60


# --------------------------------------------------------------------------
# 5. the pins above reject plausible mistakes planted in the oracle
# --------------------------------------------------------------------------
def _eos_opens_document(tokens_row, eos_id):
    is_eos = (np.asarray(tokens_row) == eos_id).astype(np.int64)
    return np.cumsum(is_eos)


def _inclusive_window(S, mask_type, tokens_row=None, eos_id=None, fixed_block_size=0, sliding_window=0):
    m = ORIG_ALLOWED(S, mask_type, tokens_row, eos_id, fixed_block_size, 0)
    if sliding_window > 0:
        i = np.arange(S)[:, None]
        j = np.arange(S)[None, :]
        m &= (i - j) <= sliding_window
    return m


def _sink_missing_from_denominator(q_bh, k_bg, mask, scale, sigma):
    return ORIG_PROBS(q_bh, k_bg, mask, scale, None)


def _scale_always_applied(head_dim, scale, sink_weights):
    return float(scale) if scale is not None else float(head_dim) ** -0.5


ORIG_ALLOWED = flex.allowed
ORIG_PROBS = flex._probabilities

MUTANTS = {
    "EOS opens the next document": ("document_ids", _eos_opens_document),
    "window bound inclusive": ("allowed", _inclusive_window),
    "sink left out of the denominator": ("_probabilities", _sink_missing_from_denominator),
    "scale applied with sink weights": ("effective_scale", _scale_always_applied),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_reject_planted_mistakes(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(flex, attr, fn)
    battery = [
        test_tiny_block_causal_by_hand,
        lambda: test_block_causal_fixed_blocks_and_window_are_sdpa_with_walked_masks(6, 4),
        test_sink_is_a_closed_form_of_the_sinkless_result,
        test_scale_is_not_applied_with_sink_weights,
        test_fixed_block_of_one_and_window_of_one_return_v,
    ]
    failed = 0
    for t in battery:
        try:
            t()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught: {name}"


@pytest.mark.parametrize("fbs,win,mask", [(0, 0, "block_causal"), (37, 11, "block_causal"), (0, 7, "causal"),
                                          (16, 0, "causal")])
def test_flop_count_of_the_generator_matches_the_oracle_mask(fbs, win, mask):
    w = W.FlexWorkload("count", 2, 300, 4, 2, 8, mask, docs=(5, 60), fixed_block_size=fbs, sliding_window=win)
    x = W.make_flex_inputs(w)
    E = sum(int(flex.allowed(w.seq, mask, x["tokens"][b].numpy(), w.eos_id, fbs, win).sum()) for b in range(2))
    assert W.flex_allowed_counts(w, x) == E * w.heads_q
