"""The forward entry point that allocates nothing.

Some callers cannot allocate device memory (they only get input and output
buffers from their host framework, or may not call cudaMalloc because it can
synchronise the device). inkling_rel_attn_fwd_noalloc serves them with scratch
held in a static device array inside the library. This file runs last (pytest
collects it after the others) and checks, through the C ABI, that two calls in
a row agree with the ordinary workspace-taking forward, that a call leaves the
device's free memory and PyTorch's allocation count unchanged, and that the
entry point's own device error word reads back clean.
"""
import pytest
import torch

from learned_relative_gqa_b200 import binding
from learned_relative_gqa_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from learned_relative_gqa_b200 import build
    build.build()


def test_noalloc_forward_matches_workspace_forward_twice():
    w = U.custom("noalloc", 2, 520, 8, 2, 128, 0, 256, docs=(60, 400), pad=(0, 40))
    x = W.make_inputs(w, "cuda")
    ref_out, ref_lse = U.gpu_forward(x)
    dims = binding.make_dims(x["q"], x["k"], x["profiles"], x["window"], x["query_offset"])
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        torch.cuda.synchronize()
        # the first call loads the library's module and looks its scratch up; from the
        # second on, a call must not change the device's free memory at all
        free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        st = binding.inkling_rel_attn_fwd_noalloc(dims, x["q"], x["k"], x["v"], x["profiles"], x["sink"],
                                                  x["valid"], x["key_valid"], x["positions"], x["key_positions"],
                                                  out, lse)
        assert st == binding.INKLING_OK
        torch.cuda.synchronize()
        if call > 0:
            assert torch.cuda.mem_get_info()[0] == free0, "the no-allocation forward changed free device memory"
            assert torch.cuda.memory_allocated() == alloc0
        assert binding.inkling_rel_attn_fwd_noalloc_last_device_error() == binding.INKLING_OK
        U.assert_out_close(out.cpu().numpy(), ref_out.cpu().double().numpy(), "noalloc out")
        U.assert_lse_close(lse.cpu().numpy(), ref_lse.cpu().double().numpy(), "noalloc lse")


def test_noalloc_forward_rejects_problems_beyond_its_scratch():
    x = W.make_inputs(U.custom("small", 1, 128, 2, 1, 64, 0, 8), "cuda")
    big = binding.Dims(64, 16384, 16384, 2, 1, 64, 8, 0, 0)   # about 9 MB of scratch needed
    st = binding.inkling_rel_attn_fwd_noalloc(big, x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"],
                                              x["key_valid"], x["positions"], x["key_positions"], x["q"], x["q"])
    assert st == binding.INKLING_ERR_UNSUPPORTED
