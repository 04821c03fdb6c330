"""GPU forward vs the FP64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

from learned_relative_gqa_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu

SMALL = [
    U.custom("ragged_docs_pad", 2, 200, 4, 2, 128, 0, 64, docs=(20, 90), pad=(0, 30)),
    U.custom("odd_group_d64_window", 1, 130, 6, 2, 64, 50, 48, docs=(10, 60)),
    U.custom("mha_no_profiles", 1, 256, 2, 2, 128, 0, 0, pad=(0, 40)),
    U.custom("query_offset_slice", 2, 160, 4, 1, 128, 0, 96, docs=(30, 150), seq_k=384, query_offset=200),
    U.custom("single_token", 1, 1, 2, 1, 64, 0, 8),
    U.custom("window_one", 1, 300, 4, 2, 128, 1, 8),
    U.custom("extent_beyond_seq", 1, 192, 4, 4, 64, 0, 256, docs=(40, 100)),
    U.custom("local_small", 1, 640, 8, 2, 128, 256, 256, pad=(0, 127)),
    U.custom("many_short_docs", 1, 384, 4, 2, 128, 0, 32, docs=(1, 7)),
    U.custom("d64_pairs_long", 1, 1000, 4, 2, 64, 0, 200, docs=(100, 700), pad=(0, 50)),
    # no profiles, D 128, paired heads
    U.custom("no_profiles_pairs", 2, 300, 8, 2, 128, 0, 0, docs=(30, 250), pad=(0, 20)),
    U.custom("no_profiles_window_long", 1, 1100, 4, 2, 128, 200, 0, docs=(100, 900), pad=(0, 60)),
    U.custom("no_profiles_offset_slice", 2, 160, 4, 1, 128, 0, 0, docs=(30, 150), seq_k=384, query_offset=200),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from learned_relative_gqa_b200 import build
    build.build()


def check_full(x):
    out, lse = U.gpu_forward(x)
    torch.cuda.synchronize()
    h = U.to_host(x)
    o_ref, l_ref, _ = U.oracle_forward(h)
    U.assert_out_close(out.cpu().numpy(), o_ref)
    U.assert_lse_close(lse.cpu().numpy(), l_ref)
    return out, lse


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_forward_small_shapes(w):
    check_full(W.make_inputs(w, "cuda"))


def test_forward_pr1_ref_full():
    check_full(W.make_inputs(W.BY_NAME["pr1_ref"], "cuda"))


def test_forward_local_layer_full():
    check_full(W.make_inputs(W.BY_NAME["local"], "cuda"))


def test_forward_extreme_sinks():
    w = U.custom("sinks", 1, 256, 4, 2, 128, 0, 64, docs=(30, 200))
    x = W.make_inputs(w, "cuda")
    s = x["sink"]
    s[0, ::7, 0] = float("-inf")
    s[0, ::5, 1] = 40.0
    s[0, ::3, 2] = -40.0
    check_full(x)


@pytest.mark.parametrize("name,nrows", [("packed", 768), ("long", 768), ("train", 768)])
def test_forward_full_size_sampled_rows(name, nrows):
    w = W.BY_NAME[name]
    x = W.make_inputs(w, "cuda")
    out, lse = U.gpu_forward(x)
    torch.cuda.synchronize()
    rows = U.sample_rows(x, nrows)
    h = U.to_host(x)
    o_ref, l_ref, _ = U.oracle_forward(h, rows=rows)
    B, S, Hq, D = x["q"].shape
    o_gpu = out.cpu().numpy().reshape(-1, D)[rows]
    l_gpu = lse.cpu().numpy().reshape(-1)[rows]
    U.assert_out_close(o_gpu, o_ref.reshape(-1, D)[rows])
    U.assert_lse_close(l_gpu, l_ref.reshape(-1)[rows])
    # properties of every row: finite, and padded rows give out = 0, lse = sink
    o_all = out.view(B, S, Hq, D)
    assert torch.isfinite(o_all).all()
    inval = ~x["valid"].bool()
    if inval.any():
        assert (o_all[inval] == 0).all()
        assert torch.equal(lse[inval], x["sink"][inval])


def test_forward_is_deterministic():
    x = W.make_inputs(U.custom("det", 2, 384, 8, 2, 128, 0, 128, docs=(50, 300)), "cuda")
    a = U.gpu_forward(x)
    b = U.gpu_forward(x)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_forward_empty_batch_is_noop():
    from learned_relative_gqa_b200 import binding
    x = W.make_inputs(U.custom("empty", 1, 128, 4, 2, 128, 0, 64), "cuda")
    out, lse = binding.forward(
        x["q"][:, :0].contiguous(), x["k"], x["v"], x["profiles"][:, :, :0].contiguous(),
        x["sink"][:, :0].contiguous(), x["valid"][:, :0].contiguous(), x["key_valid"],
        x["positions"][:, :0].contiguous(), x["key_positions"], window=0, query_offset=0)
    assert out.numel() == 0 and lse.numel() == 0


def test_forward_default_masks_and_positions():
    # key_valid, positions and key_positions left to their defaults: one document, keys = queries
    from learned_relative_gqa_b200 import binding
    w = U.custom("defaults", 2, 192, 4, 2, 128, 64, 64)
    x = W.make_inputs(w, "cuda")
    out, lse = binding.forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], None, None, None,
                               window=64)
    torch.cuda.synchronize()
    h = U.to_host(x)
    import oracle
    o_ref, l_ref, _ = oracle.forward(h["q"], h["k"], h["v"], h["profiles"], h["sink"], h["valid"], window=64)
    U.assert_out_close(out.cpu().numpy(), o_ref)
    U.assert_lse_close(lse.cpu().numpy(), l_ref)


@pytest.mark.parametrize("seq_k", [523, 512])
def test_forward_key_span_starts_and_ends_inside_words(seq_k):
    """Key streams whose valid span starts at column 0, 5, 16 or 37 and ends at a
    random column, with rows that start on and off 16-byte boundaries: the key span
    (first / last valid key of each batch row) is found for every alignment."""
    from learned_relative_gqa_b200 import binding
    w = U.custom(f"kspan_{seq_k}", 4, 200, 4, 2, 64, 0, 64, docs=(40, 180), pad=(0, 20), seq_k=seq_k,
                 query_offset=seq_k - 223)
    x = W.make_inputs(w, "cuda")
    for b, a in enumerate((0, 5, 16, 37)):
        x["key_valid"][b, :a] = False
    dims = binding.make_dims(x["q"], x["k"], x["profiles"], x["window"], x["query_offset"])
    ws = binding.alloc_workspace(dims, False, "cuda")
    assert binding.inkling_rel_attn_validate(dims, x["valid"], x["key_valid"], x["positions"], x["key_positions"],
                                             ws) == binding.INKLING_OK
    check_full(x)


def ramp_profiles(x, slope):
    """profiles[b, h, i, d] = slope * d rounded to BF16 (the oracle reads the same values)."""
    B, H, S, R = x["profiles"].shape
    d = torch.arange(R, device=x["profiles"].device, dtype=torch.float32)
    x["profiles"].copy_((slope * d).to(torch.bfloat16).expand(B, H, S, R))


@pytest.mark.parametrize("slope", [0.25, 0.125])
def test_forward_running_maximum_grows_every_step(slope):
    """Profiles that rise with distance make each 64-key step's row maximum exceed the
    running maximum by about 16 (slope 0.25) or 8 (slope 0.125) natural units, against a
    lazy-rescale threshold of 8 log2 units = 5.5 natural units: the
    steps visit keys from the diagonal outwards, so O is rescaled in every step after a
    row's first (including the wait for the previous PV product)."""
    w = U.custom("growing_max", 1, 320, 4, 2, 128, 0, 320, docs=(150, 300))
    x = W.make_inputs(w, "cuda")
    ramp_profiles(x, slope)
    check_full(x)
