"""GPU L2Clip vs its FP64 oracle (through the C ABI).

The output is BF16 (x's dtype): besides the FP32 arithmetic it carries the final
rounding, half a BF16 ulp of the value, which the check allows on top of 1e-5 of
the threshold-scale. Gradients: max |g - g_ref| <= 2e-2 * max |g_ref| per tensor,
as for the attention (they are FP32 sums of FP32 products, far inside that).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import l2clip as ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from learned_relative_gqa_b200 import build
    build.build()


def draw(B, S, H, D, seed, with_scale, with_tau):
    g = torch.Generator("cuda")
    g.manual_seed(seed)
    x = (torch.randn(B, S, H, D, generator=g, device="cuda")
         * torch.rand(B, S, H, 1, generator=g, device="cuda") * 3).to(torch.bfloat16)
    scale = (0.5 + torch.rand(H, D, generator=g, device="cuda")) if with_scale else None
    tau = (0.5 + 1.5 * torch.rand(B, S, generator=g, device="cuda")) if with_tau else None
    dy = torch.randn(B, S, H, D, generator=g, device="cuda")
    return x, scale, tau, dy


def f64(t):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return oracle.decode_bf16(t.cpu().view(torch.int16).numpy())
    return t.cpu().double().numpy()


CASES = [(2, 300, 8, 128, True, True, 8.0), (1, 77, 4, 64, False, True, 5.0), (3, 50, 32, 128, True, False, 10.0),
         (1, 129, 2, 128, False, False, 0.0), (2, 64, 4, 64, True, True, 1e9)]


@pytest.mark.parametrize("B,S,H,D,ws,wt,thr", CASES)
def test_l2clip_forward_backward(B, S, H, D, ws, wt, thr):
    from learned_relative_gqa_b200 import binding
    x, scale, tau, dy = draw(B, S, H, D, 11 + B * S, ws, wt)
    y = binding.l2clip_forward(x, thr, scale, tau)
    g = binding.l2clip_backward(x, dy, thr, scale, tau)
    torch.cuda.synchronize()
    y_ref = ref.forward(f64(x), f64(scale), f64(tau), thr)
    yg = f64(y)
    mag = np.maximum(np.abs(y_ref), 2.0 ** -126)
    half_ulp = 0.5 * 2.0 ** (np.floor(np.log2(mag)) - 7)
    err = np.abs(yg - y_ref) - half_ulp
    assert err.max() <= 1e-5 * max(1.0, float(np.abs(y_ref).max())), err.max()
    r = ref.backward(f64(x), f64(scale), f64(tau), thr, f64(dy))
    for name in ("dx", "dscale", "dtau"):
        if r[name] is None:
            assert g[name] is None
            continue
        got = g[name].cpu().double().numpy()
        assert np.abs(got - r[name]).max() <= 2e-2 * max(np.abs(r[name]).max(), 1e-30), name


def test_l2clip_is_deterministic():
    from learned_relative_gqa_b200 import binding
    x, scale, tau, dy = draw(2, 333, 8, 128, 5, True, True)
    a = binding.l2clip_backward(x, dy, 4.0, scale, tau)
    b = binding.l2clip_backward(x, dy, 4.0, scale, tau)
    for n in ("dx", "dscale", "dtau"):
        assert torch.equal(a[n], b[n])


def test_l2clip_full_size_q_of_the_training_shape():
    """q of the 8192-token training shape (B2 S8192 Hq32 D128): properties at every row
    (clipped rows have the threshold length, the rest are unchanged up to BF16) and the
    oracle on sampled tokens."""
    from learned_relative_gqa_b200 import binding
    x, scale, tau, dy = draw(2, 8192, 32, 128, 3, True, True)
    thr = 9.0
    y = binding.l2clip_forward(x, thr, scale, tau)
    g = binding.l2clip_backward(x, dy, thr, scale, tau)
    torch.cuda.synchronize()
    z = x.float() * scale
    n = z.norm(dim=-1)
    ny = (y.float() / tau[:, :, None, None]).norm(dim=-1)
    clipped = n > thr
    assert clipped.any() and (~clipped).any()
    assert float((ny[clipped] - thr).abs().max()) <= 0.02 * thr
    idx = torch.arange(0, 8192, 997)
    xs, ts, dys = x[:, idx], tau[:, idx], dy[:, idx]
    y_ref = ref.forward(f64(xs), f64(scale), f64(ts), thr)
    assert np.abs(f64(y[:, idx]) - y_ref).max() <= 0.02
    r = ref.backward(f64(xs), f64(scale), f64(ts), thr, f64(dys))
    assert np.abs(g["dx"][:, idx].cpu().double().numpy() - r["dx"]).max() <= 2e-2 * np.abs(r["dx"]).max()
    assert np.abs(g["dtau"][:, idx].cpu().double().numpy() - r["dtau"]).max() <= 2e-2 * np.abs(r["dtau"]).max()
    assert torch.isfinite(g["dscale"]).all()
