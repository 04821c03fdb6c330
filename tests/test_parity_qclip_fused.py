"""L2Clip of q fused into the attention kernels (inkling_rel_attn_fwd_qclip /
inkling_rel_attn_bwd_qclip) against the two FP64 oracles composed.

Reference: the L2Clip oracle clips the unclipped q x, its result is rounded to
BF16 (the dtype the clipped q has on the path, as L2Clip.forward returns x's
dtype) and fed, as q, to the attention oracle; the attention oracle's query
gradient is fed back through the L2Clip oracle's backward, which gives dx,
dscale and dtau. The kernels clip each Q tile in FP32 and round it to BF16 too,
so a clipped element may sit one BF16 rounding step away from the reference's;
the stored clipped q is checked within half a BF16 ulp of the FP64 value plus
1e-6, every other result at the parity tolerances of the unfused path.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import l2clip as clip_oracle
from learned_relative_gqa_b200 import binding
from learned_relative_gqa_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from learned_relative_gqa_b200 import build
    build.build()


CASES = [
    # (workload, learned scales, length scaling, threshold)
    (U.custom("qclip_train_like", 2, 300, 8, 2, 128, 64, 64, docs=(30, 250), pad=(0, 20)), True, True, 9.0),
    (U.custom("qclip_plain_d64", 1, 200, 4, 2, 64, 0, 32, docs=(20, 150)), False, False, 5.0),
    (U.custom("qclip_zero_threshold", 1, 130, 4, 4, 128, 0, 16), True, False, 0.0),
]


def _bf16_f64(t):
    return oracle.decode_bf16(t.cpu().view(torch.int16).numpy())


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_fused_qclip_matches_the_composed_oracles(case):
    w, with_scale, with_tau, thr = case
    x = W.make_inputs(w, "cuda", with_dout=True)
    B, S, Hq, D = x["q"].shape
    g = torch.Generator("cuda")
    g.manual_seed(4242)
    # the unclipped q: per-vector lengths spread over both sides of the threshold
    xq = (x["q"].float() * (0.2 + 1.6 * torch.rand(B, S, Hq, 1, generator=g, device="cuda"))).to(torch.bfloat16)
    scale = (0.5 + torch.rand(Hq, D, generator=g, device="cuda")) if with_scale else None
    tau = (0.5 + 1.5 * torch.rand(B, S, generator=g, device="cuda")) if with_tau else None
    kw = dict(threshold=thr, clip_scale=scale, tau=tau, window=x["window"], query_offset=x["query_offset"])
    out, lse, qc = binding.forward_qclip(xq, x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                                         x["positions"], x["key_positions"], **kw)
    gr = binding.backward_qclip(xq, qc, x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                                x["positions"], x["key_positions"], out, lse, x["dout"], **kw)
    torch.cuda.synchronize()

    xh = _bf16_f64(xq)
    sc = None if scale is None else scale.cpu().double().numpy()
    ta = None if tau is None else tau.cpu().double().numpy()
    y = clip_oracle.forward(xh, sc, ta, thr)
    # the clipped q as stored: within half a BF16 ulp of the FP64 value
    mag = np.maximum(np.abs(y), 2.0 ** -126)
    half_ulp = 0.5 * 2.0 ** (np.floor(np.log2(mag)) - 7)
    assert np.all(np.abs(_bf16_f64(qc) - y) <= half_ulp + 1e-6), "clipped q"
    # attention on the oracle's own BF16 rounding of the clipped q
    h = U.to_host(x)
    h["q"] = _bf16_f64(torch.from_numpy(y).to(torch.bfloat16))
    o_ref, l_ref, _ = U.oracle_forward(h)
    U.assert_out_close(out.cpu().numpy(), o_ref)
    U.assert_lse_close(lse.cpu().numpy(), l_ref)
    ref = U.oracle_backward(h)
    for n in ("dk", "dv", "dprofiles", "dsink"):
        U.assert_grad_close(gr[n].cpu().numpy(), ref[n], n)
    back = clip_oracle.backward(xh, sc, ta, thr, ref["dq"])
    U.assert_grad_close(gr["dx"].cpu().numpy(), back["dx"], "dx")
    if with_scale:
        U.assert_grad_close(gr["dclip_scale"].cpu().numpy(), back["dscale"], "dclip_scale")
    else:
        assert gr["dclip_scale"] is None
    if with_tau:
        U.assert_grad_close(gr["dtau"].cpu().numpy(), back["dtau"], "dtau")
    else:
        assert gr["dtau"] is None


def test_fused_qclip_equals_the_separate_passes():
    """The fused path against the standalone L2Clip kernels around the unfused attention
    kernels, all on the GPU: the same clipped q bit for bit where the two FP32 roundings
    agree, and results within the parity tolerances."""
    w = CASES[0][0]
    x = W.make_inputs(w, "cuda", with_dout=True)
    B, S, Hq, D = x["q"].shape
    g = torch.Generator("cuda")
    g.manual_seed(7)
    xq = (x["q"].float() * (0.2 + 1.6 * torch.rand(B, S, Hq, 1, generator=g, device="cuda"))).to(torch.bfloat16)
    scale = 0.5 + torch.rand(Hq, D, generator=g, device="cuda")
    tau = 0.5 + 1.5 * torch.rand(B, S, generator=g, device="cuda")
    kw = dict(window=x["window"], query_offset=x["query_offset"])
    out, lse, qc = binding.forward_qclip(xq, x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                                         x["positions"], x["key_positions"], threshold=9.0, clip_scale=scale,
                                         tau=tau, **kw)
    q2 = binding.l2clip_forward(xq, 9.0, scale, tau)
    torch.cuda.synchronize()
    differ = (qc.view(torch.int16) != q2.view(torch.int16)).float().mean().item()
    assert differ < 1e-3, f"{differ:.2e} of the clipped elements differ"
    o2, l2 = binding.forward(q2, x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                             x["positions"], x["key_positions"], **kw)
    torch.cuda.synchronize()
    assert float((out - o2).abs().max()) <= U.OUT_MAX and float((lse - l2).abs().max()) <= U.LSE_TOL


def test_fused_qclip_full_size_matches_the_separate_passes():
    """The training shape the bench times (B2 S8192 Hq32 Hkv4 D128, window 1024, R 1024,
    documents), with learned scales, tau and threshold 9: the fused kernels against the
    standalone L2Clip kernels around the unfused attention kernels (each checked against
    its oracle in the tests above and in the attention parity tests), compared on the GPU
    at the parity tolerances; the stored clipped q bit for bit except where the two FP32
    evaluations round to neighbouring BF16 values."""
    w = W.BY_NAME["train"]
    x = W.make_inputs(w, "cuda", with_dout=True)
    B, S, Hq, D = x["q"].shape
    g = torch.Generator("cuda")
    g.manual_seed(11)
    xq = (x["q"].float() * (0.2 + 1.6 * torch.rand(B, S, Hq, 1, generator=g, device="cuda"))).to(torch.bfloat16)
    scale = 0.5 + torch.rand(Hq, D, generator=g, device="cuda")
    tau = 0.5 + 1.5 * torch.rand(B, S, generator=g, device="cuda")
    a = (x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"], x["positions"], x["key_positions"])
    kw = dict(window=x["window"], query_offset=x["query_offset"])
    out, lse, qc = binding.forward_qclip(xq, *a, threshold=9.0, clip_scale=scale, tau=tau, **kw)
    gf = binding.backward_qclip(xq, qc, *a, out, lse, x["dout"], threshold=9.0, clip_scale=scale, tau=tau, **kw)
    q2 = binding.l2clip_forward(xq, 9.0, scale, tau)
    o2, l2 = binding.forward(q2, *a, **kw)
    gs = binding.backward(q2, *a, o2, l2, x["dout"], **kw)
    back = binding.l2clip_backward(xq, gs["dq"], 9.0, scale, tau)
    torch.cuda.synchronize()

    differ = (qc.view(torch.int16) != q2.view(torch.int16)).float().mean().item()
    assert differ < 1e-3, f"{differ:.2e} of the clipped elements differ"

    def close(a_, b_, tol, what, relative):
        assert bool(torch.isfinite(a_).all()), f"{what}: non-finite values"
        err = float((a_.double() - b_.double()).abs().max())
        bound = tol * max(float(b_.abs().max()), 1e-30) if relative else tol
        assert err <= bound, f"{what}: max abs err {err:.3e} > {bound:.3e}"

    close(out, o2, U.OUT_MAX, "out", False)
    assert float((out.double() - o2.double()).abs().mean()) <= U.OUT_MEAN
    close(lse, l2, U.LSE_TOL, "lse", False)
    for n_ in ("dk", "dv", "dprofiles", "dsink"):
        close(gf[n_], gs[n_], U.GRAD_REL, n_, True)
    close(gf["dx"], back["dx"], U.GRAD_REL, "dx", True)
    close(gf["dclip_scale"], back["dscale"], U.GRAD_REL, "dclip_scale", True)
    close(gf["dtau"], back["dtau"], U.GRAD_REL, "dtau", True)
