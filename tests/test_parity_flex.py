"""GPU generic FlexAttention variant vs its FP64 oracle (through the C ABI).

Tolerances as for the learned-relative path: lse within 1e-3, gradients
max |g - g_ref| <= 2e-2 * max |g_ref|, outputs max |err| <= 1e-2 and mean
|err| <= 1e-3 -- but this variant returns its output in BF16 (q's dtype, as the
FlexAttention page states), and rounding the result to BF16 alone moves it by
up to half a BF16 ulp (2^-9 relative: 0.0078 for outputs in [2, 4)). The output
check therefore takes that half ulp of the reference value off each error
before applying the two bounds.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import flex as flex_oracle
from learned_relative_gqa_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from learned_relative_gqa_b200 import build
    build.build()


def _f64(t):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return oracle.decode_bf16(t.cpu().view(torch.int16).numpy())
    return t.cpu().double().numpy()


def kw_of(x):
    return dict(mask_type=x["mask_type"], eos_id=x["eos_id"], fixed_block_size=x["fixed_block_size"],
                sliding_window=x["sliding_window"], scale=x["scale"], enable_gqa=x["enable_gqa"])


def gpu_fwd(x):
    from learned_relative_gqa_b200 import binding
    return binding.flex_forward(x["q"], x["k"], x["v"], x["sink_weights"], x["tokens"], **kw_of(x))


def gpu_bwd(x, out, lse):
    from learned_relative_gqa_b200 import binding
    return binding.flex_backward(x["q"], x["k"], x["v"], out, lse, x["dout"], x["sink_weights"], x["tokens"],
                                 **kw_of(x))


def oracle_fwd(x, sl=slice(None), heads=slice(None), kv_heads=slice(None)):
    sw = x["sink_weights"]
    return flex_oracle.forward(_f64(x["q"][sl, heads]), _f64(x["k"][sl, kv_heads]), _f64(x["v"][sl, kv_heads]),
                               None if sw is None else _f64(sw[heads]), x["tokens"][sl].cpu().numpy(), **kw_of(x))


def oracle_bwd(x, sl=slice(None), heads=slice(None), kv_heads=slice(None)):
    sw = x["sink_weights"]
    return flex_oracle.backward(_f64(x["q"][sl, heads]), _f64(x["k"][sl, kv_heads]), _f64(x["v"][sl, kv_heads]),
                                None if sw is None else _f64(sw[heads]), x["tokens"][sl].cpu().numpy(),
                                dout=_f64(x["dout"][sl, heads]), **kw_of(x))


def assert_bf16_out_close(out_gpu, out_ref):
    o = np.asarray(out_gpu, dtype=np.float64)
    assert np.all(np.isfinite(o)), "out: non-finite values"
    mag = np.maximum(np.abs(out_ref), 2.0 ** -126)
    half_ulp = 0.5 * 2.0 ** (np.floor(np.log2(mag)) - 7)   # BF16: 8 significant bits
    err = np.maximum(np.abs(o - out_ref) - half_ulp, 0.0)
    assert err.max() <= U.OUT_MAX, f"out: max abs err beyond the BF16 rounding {err.max():.3e} > {U.OUT_MAX}"
    assert err.mean() <= U.OUT_MEAN, f"out: mean abs err beyond the BF16 rounding {err.mean():.3e} > {U.OUT_MEAN}"


def assert_grad_close(g, ref, what):
    g = np.asarray(g, dtype=np.float64)
    scale = float(np.abs(ref).max())
    err = float(np.abs(g - ref).max())
    assert err <= U.GRAD_REL * max(scale, 1e-30), f"{what}: max err {err:.3e} vs max |ref| {scale:.3e}"


CASES = [
    W.FlexWorkload("blockcausal_gqa_sinks", 2, 600, 8, 2, 128, "block_causal", docs=(20, 300)),
    W.FlexWorkload("causal_mha_d64_scale", 1, 333, 4, 4, 64, "causal", sink=False, scale=0.2),
    W.FlexWorkload("fixed_blocks_window", 2, 517, 4, 1, 128, "block_causal", docs=(30, 400),
                   fixed_block_size=100, sliding_window=70),
    W.FlexWorkload("causal_fixed_blocks_d64", 1, 256, 2, 1, 64, "causal", fixed_block_size=64),
    W.FlexWorkload("many_tiny_docs", 1, 300, 4, 2, 128, "block_causal", docs=(1, 5), sink=False),
    W.FlexWorkload("window_one", 1, 200, 2, 2, 128, "causal", sliding_window=1),
    W.FlexWorkload("scale_ignored_with_sinks", 1, 192, 4, 2, 128, "causal", scale=0.05),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_flex_forward_and_backward_small(w):
    x = W.make_flex_inputs(w, "cuda")
    out, lse = gpu_fwd(x)
    g = gpu_bwd(x, out, lse)
    torch.cuda.synchronize()
    assert out.dtype == torch.bfloat16 and out.shape == x["q"].shape and lse.shape == x["q"].shape[:3]
    o_ref, l_ref = oracle_fwd(x)
    assert_bf16_out_close(out.float().cpu().numpy(), o_ref)
    U.assert_lse_close(lse.cpu().numpy(), l_ref)
    r = oracle_bwd(x)
    for name in ("dq", "dk", "dv"):
        assert_grad_close(g[name].cpu().numpy(), r[name], name)
    if w.sink:
        assert_grad_close(g["dsink_weights"].cpu().numpy(), r["dsink_weights"], "dsink_weights")
    else:
        assert g["dsink_weights"] is None


def test_flex_is_deterministic():
    x = W.make_flex_inputs(CASES[0], "cuda")
    a = gpu_fwd(x)
    b = gpu_fwd(x)
    ga = gpu_bwd(x, *a)
    gb = gpu_bwd(x, *b)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    for n in ("dq", "dk", "dv", "dsink_weights"):
        assert torch.equal(ga[n], gb[n]), n


def test_flex_matches_the_learned_relative_path_without_profiles():
    """The same problem through the learned-relative ABI (R = 0, positions restarting at
    each document, sink broadcast to every row): identical FP32 statistics."""
    from learned_relative_gqa_b200 import binding
    w = CASES[2]
    x = W.make_flex_inputs(w, "cuda")
    out, lse = gpu_fwd(x)
    B, Hq, S, D = x["q"].shape
    tok = x["tokens"].cpu()
    pos = torch.zeros(B, S, dtype=torch.int32)
    for b in range(B):
        start = 0
        for i in range(S):
            if i > 0 and (int(tok[b, i - 1]) == w.eos_id or i % w.fixed_block_size == 0):
                start = i
            pos[b, i] = i - start
    pos = pos.cuda()
    valid = torch.ones(B, S, dtype=torch.bool, device="cuda")
    sink = x["sink_weights"].view(1, 1, Hq).expand(B, S, Hq).contiguous()
    o2, l2 = binding.forward(x["q"].transpose(1, 2).contiguous(), x["k"].transpose(1, 2).contiguous(),
                             x["v"].transpose(1, 2).contiguous(), torch.empty(B, Hq, S, 0, dtype=torch.bfloat16,
                                                                              device="cuda"),
                             sink, valid, valid, pos, pos, window=w.sliding_window)
    torch.cuda.synchronize()
    assert torch.equal(lse, l2.transpose(1, 2))
    assert torch.equal(out, o2.transpose(1, 2).to(torch.bfloat16))


@pytest.mark.parametrize("pick", [(0, 0), (3, 5)])
def test_flex_full_size_packed_sampled_groups(pick):
    """The packed-documents shape (B4 S4096 Hq32 Hkv8, EOS-delimited documents, per-head
    sinks), checked on one batch row and one KV head group against the oracle."""
    w = W.FLEX_BY_NAME["flex_packed"]
    x = W.make_flex_inputs(w, "cuda")
    out, lse = gpu_fwd(x)
    g = gpu_bwd(x, out, lse)
    torch.cuda.synchronize()
    b, grp = pick
    G = w.heads_q // w.heads_kv
    sl, hs, ks = slice(b, b + 1), slice(grp * G, (grp + 1) * G), slice(grp, grp + 1)
    o_ref, l_ref = oracle_fwd(x, sl, hs, ks)
    assert_bf16_out_close(out[sl, hs].float().cpu().numpy(), o_ref)
    U.assert_lse_close(lse[sl, hs].cpu().numpy(), l_ref)
    r = oracle_bwd(x, sl, hs, ks)
    assert_grad_close(g["dq"][sl, hs].cpu().numpy(), r["dq"], "dq")
    assert_grad_close(g["dk"][sl, ks].cpu().numpy(), r["dk"], "dk")
    assert_grad_close(g["dv"][sl, ks].cpu().numpy(), r["dv"], "dv")
    assert torch.isfinite(g["dsink_weights"]).all()
