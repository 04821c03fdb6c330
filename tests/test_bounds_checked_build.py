"""The attention kernels built with every shared- and global-memory index checked.

``-DINKLING_BOUNDS_CHECK`` compiles, next to the product library, a variant in
which each shared-memory, global-memory and tensor-copy access of the forward,
dK/dV and dQ kernels first tests its index against the extent of its buffer; an
index outside records a code in the workspace's device error word and the
access is skipped (nothing traps). The small and odd shapes below (a ragged tail
of every tile size, one-token rows, odd GQA groups, windows of one, a query
slice against global keys, the generic variant's [B, H, S, D] strides and BF16
output) run through it, forward and backward; every call must leave the error
word clean and still match the FP64 oracle at the parity tolerances.
"""
import pytest
import torch

from learned_relative_gqa_b200 import binding
from learned_relative_gqa_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu

CASES = [
    U.custom("bc_ragged", 2, 200, 4, 2, 128, 0, 64, docs=(10, 90), pad=(0, 30)),
    U.custom("bc_odd_group", 1, 129, 3, 1, 64, 17, 24, docs=(5, 60)),
    U.custom("bc_one_token", 1, 1, 2, 2, 64, 0, 8),
    U.custom("bc_window_one", 2, 70, 8, 2, 128, 1, 16, pad=(0, 20)),
    U.custom("bc_slice", 1, 96, 4, 2, 128, 40, 32, docs=(20, 80), seq_k=224, query_offset=128),
]


@pytest.fixture(scope="module")
def checked():
    from learned_relative_gqa_b200 import build
    path = build.BOUNDS_CHECK_LIB_PATH
    if build.stale(path):
        build.build(defines=("INKLING_BOUNDS_CHECK",), out_path=path)
    saved = binding._lib
    binding._lib = None
    binding.load(path)
    yield
    binding._lib = saved


def _clean(ws):
    torch.cuda.synchronize()
    assert binding.inkling_rel_attn_last_device_error(ws) == binding.INKLING_OK, "an index left its buffer"


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_checked_build_records_no_out_of_bounds_index(checked, w):
    x = W.make_inputs(w, "cuda", with_dout=True)
    dims = binding.make_dims(x["q"], x["k"], x["profiles"], x["window"], x["query_offset"])
    wsf = binding.alloc_workspace(dims, False, x["q"].device)
    out, lse = binding.forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                               x["positions"], x["key_positions"], window=x["window"],
                               query_offset=x["query_offset"], workspace=wsf)
    _clean(wsf)
    wsb = binding.alloc_workspace(dims, True, x["q"].device)
    g = binding.backward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                         x["positions"], x["key_positions"], out, lse, x["dout"], window=x["window"],
                         query_offset=x["query_offset"], workspace=wsb)
    _clean(wsb)
    h = U.to_host(x)
    o_ref, l_ref, _ = U.oracle_forward(h)
    U.assert_out_close(out.cpu().numpy(), o_ref)
    U.assert_lse_close(lse.cpu().numpy(), l_ref)
    ref = U.oracle_backward(h)
    for n in ("dq", "dk", "dv", "dprofiles", "dsink"):
        U.assert_grad_close(g[n].cpu().numpy(), ref[n], n)


def test_checked_build_generic_variant(checked):
    from tests import test_parity_flex as F
    wf = W.FlexWorkload("bc_flex", 2, 150, 4, 2, 64, "block_causal", docs=(10, 70), fixed_block_size=48,
                        sliding_window=33)
    x = W.make_flex_inputs(wf, "cuda")
    dims = binding.make_flex_dims(x["q"], x["k"], **F.kw_of(x))
    wsf = torch.empty(binding.inkling_flex_attn_workspace_size(dims, False), dtype=torch.uint8, device="cuda")
    out = torch.empty(x["q"].shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(x["q"].shape[:3], dtype=torch.float32, device="cuda")
    binding.inkling_flex_attn_fwd(dims, x["q"], x["k"], x["v"], x["sink_weights"], x["tokens"], out, lse, wsf)
    _clean(wsf)
    wsb = torch.empty(binding.inkling_flex_attn_workspace_size(dims, True), dtype=torch.uint8, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty(x["q"].shape, **f32), torch.empty(x["k"].shape, **f32), torch.empty(x["v"].shape, **f32)
    dsw = torch.empty(x["sink_weights"].shape, **f32)
    binding.inkling_flex_attn_bwd(dims, x["q"], x["k"], x["v"], x["sink_weights"], x["tokens"], out, lse, x["dout"],
                                  dq, dk, dv, dsw, wsb)
    _clean(wsb)
    o_ref, l_ref = F.oracle_fwd(x)
    F.assert_bf16_out_close(out.float().cpu().numpy(), o_ref)
    U.assert_lse_close(lse.cpu().numpy(), l_ref)
    r = F.oracle_bwd(x)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv), ("dsink_weights", dsw)):
        F.assert_grad_close(g.cpu().numpy(), r[name], name)
