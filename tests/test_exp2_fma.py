"""Accuracy of the FMA-pipe power of two the forward kernel uses for a share of its
softmax exponentials (range reduction + fitted cubic), against exp2 in FP64."""
import numpy as np
import pytest
import torch

from learned_relative_gqa_b200 import binding

pytestmark = pytest.mark.gpu


def test_exp2_fma_relative_error_over_the_softmax_range():
    # the softmax arguments lie in [-inf, 8]; below -125 the result is clamped
    grid = np.linspace(-125.0, 9.0, 200001)
    rng = np.random.default_rng(7)
    extra = np.concatenate([rng.uniform(-125.0, 9.0, 50000), np.arange(-125, 10) + 0.5, np.arange(-125, 10)])
    t = torch.tensor(np.concatenate([grid, extra]), dtype=torch.float32, device="cuda")
    out = torch.empty_like(t)
    binding.inkling_rel_attn_selftest_exp2(t, out)
    torch.cuda.synchronize()
    tv = t.cpu().double().numpy()
    got = out.cpu().double().numpy()
    ref = np.exp2(tv)
    rel = np.abs(got - ref) / ref
    assert np.all(np.isfinite(got))
    assert rel.max() < 1.0e-4, f"max relative error {rel.max():.3e} at t = {tv[np.argmax(rel)]}"


def test_exp2_fma_clamps_very_negative_arguments():
    t = torch.tensor([-126.0, -1000.0, float("-inf"), -125.0], dtype=torch.float32, device="cuda")
    out = torch.empty_like(t)
    binding.inkling_rel_attn_selftest_exp2(t, out)
    torch.cuda.synchronize()
    got = out.cpu().double().numpy()
    assert np.all(got > 0) and np.all(got < 2.0 ** -124)


def test_exp2_fma_odd_length_and_empty():
    t = torch.tensor([0.0, 1.0, -1.0], dtype=torch.float32, device="cuda")
    out = torch.full_like(t, -1.0)
    binding.inkling_rel_attn_selftest_exp2(t, out)
    torch.cuda.synchronize()
    np.testing.assert_allclose(out.cpu().numpy(), [1.0, 2.0, 0.5], rtol=1e-4)
    e = torch.empty(0, dtype=torch.float32, device="cuda")
    binding.inkling_rel_attn_selftest_exp2(e, e)
