"""Pins for the FP64 oracle of L2Clip (CPU only): a case worked by hand,
closed-form properties of clipping to a ball, torch autograd of a separately
written formulation, finite differences, and planted mistakes the pins reject."""
import math

import numpy as np
import pytest
import torch

from oracle import l2clip


def draw(B=2, S=9, H=3, D=8, seed=0, spread=2.0):
    g = np.random.default_rng(seed)
    x = g.standard_normal((B, S, H, D)) * g.uniform(0.1, spread, (B, S, H, 1))
    scale = g.uniform(0.5, 1.5, (H, D))
    tau = g.uniform(0.5, 2.0, (B, S))
    dy = g.standard_normal((B, S, H, D))
    return x, scale, tau, dy


def test_hand_case():
    # (3, 4) has length 5: threshold 1 gives (0.6, 0.8); threshold 10 leaves it; tau 2 doubles
    x = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    np.testing.assert_allclose(l2clip.forward(x, None, None, 1.0).reshape(-1), [0.6, 0.8], rtol=1e-15)
    np.testing.assert_array_equal(l2clip.forward(x, None, None, 10.0), x)
    np.testing.assert_allclose(l2clip.forward(x, None, np.array([[2.0]]), 1.0).reshape(-1), [1.2, 1.6], rtol=1e-15)
    # learned scales before the clip: (3, 4) * (1/3, 1/4) = (1, 1), length sqrt 2 > 1
    y = l2clip.forward(x, np.array([[1 / 3, 1 / 4]]), None, 1.0).reshape(-1)
    np.testing.assert_allclose(y, [1 / math.sqrt(2), 1 / math.sqrt(2)], rtol=1e-15)


def test_clipped_vectors_have_the_threshold_length_and_keep_their_direction():
    x, scale, _, _ = draw()
    t = 1.3
    y = l2clip.forward(x, scale, None, t)
    z = x * scale
    nz = np.linalg.norm(z, axis=-1)
    ny = np.linalg.norm(y, axis=-1)
    out = nz > t
    assert out.any() and (~out).any()
    np.testing.assert_allclose(ny[out], t, rtol=1e-14)
    np.testing.assert_array_equal(y[~out], z[~out])
    cos = (y * z).sum(-1) / (ny * nz)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-14)


def test_length_scaling_multiplies_after_the_clip():
    x, scale, tau, _ = draw()
    a = l2clip.forward(x, scale, tau, 0.9)
    b = l2clip.forward(x, scale, None, 0.9) * tau[:, :, None, None]
    np.testing.assert_allclose(a, b, rtol=1e-15)
    assert np.linalg.norm(a, axis=-1).max() <= 0.9 * tau.max() * (1 + 1e-14)


def torch_reference(x, scale, tau, t):
    z = x * scale
    n = torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    y = torch.where(n > t, z * (t / n), z)
    return y * tau[:, :, None, None]


def test_backward_matches_autograd():
    x, scale, tau, dy = draw(seed=3)
    xs = [torch.tensor(a, requires_grad=True) for a in (x, scale, tau)]
    (torch_reference(*xs, 1.1) * torch.tensor(dy)).sum().backward()
    g = l2clip.backward(x, scale, tau, 1.1, dy)
    np.testing.assert_allclose(l2clip.forward(x, scale, tau, 1.1),
                               torch_reference(*[torch.tensor(a) for a in (x, scale, tau)], 1.1).numpy(), rtol=1e-14)
    for name, t in (("dx", xs[0]), ("dscale", xs[1]), ("dtau", xs[2])):
        np.testing.assert_allclose(g[name], t.grad.numpy(), rtol=1e-11, atol=1e-13, err_msg=name)


def test_backward_finite_differences():
    x, scale, tau, dy = draw(B=1, S=3, H=2, D=4, seed=7)
    g = l2clip.backward(x, scale, tau, 0.8, dy)

    def loss(xx, ss, tt):
        return float((l2clip.forward(xx, ss, tt, 0.8) * dy).sum())

    h = 1e-6
    for arr_i, key in ((0, "dx"), (1, "dscale"), (2, "dtau")):
        args = [x, scale, tau]
        base = args[arr_i]
        for idx in np.ndindex(base.shape):
            p = [a.copy() for a in args]
            m = [a.copy() for a in args]
            p[arr_i][idx] += h
            m[arr_i][idx] -= h
            fd = (loss(*p) - loss(*m)) / (2 * h)
            assert abs(fd - g[key][idx]) <= 1e-6 * max(1.0, abs(g[key][idx])), (key, idx, fd, g[key][idx])


def test_without_scale_or_tau():
    x, _, _, dy = draw(seed=11)
    y = l2clip.forward(x, None, None, 1.0)
    assert np.linalg.norm(y, axis=-1).max() <= 1.0 + 1e-14
    g = l2clip.backward(x, None, None, 1.0, dy)
    assert g["dscale"] is None and g["dtau"] is None


# planted mistakes
def _clip_to_unit(x, scale, tau, threshold):            # forgets the threshold
    return ORIG_FWD(x, scale, tau, 1.0)


def _tau_before_clip(x, scale, tau, threshold):           # scales the length, then clips
    xt = np.asarray(x) * (1.0 if tau is None else np.asarray(tau)[:, :, None, None])
    return ORIG_FWD(xt, scale, None, threshold)


def _scale_after_clip(x, scale, tau, threshold):          # learned scale after the clip
    y = ORIG_FWD(x, None, tau, threshold)
    return y * (1.0 if scale is None else np.asarray(scale)[None, None])


ORIG_FWD = l2clip.forward


@pytest.mark.parametrize("mut", [_clip_to_unit, _tau_before_clip, _scale_after_clip])
def test_pins_reject_planted_mistakes(mut, monkeypatch):
    monkeypatch.setattr(l2clip, "forward", mut)
    failed = 0
    for t in (test_hand_case, test_clipped_vectors_have_the_threshold_length_and_keep_their_direction,
              test_length_scaling_multiplies_after_the_clip, test_backward_matches_autograd):
        try:
            t()
        except AssertionError:
            failed += 1
    assert failed > 0
