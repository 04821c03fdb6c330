"""GPU backward vs the FP64 oracle (through the C ABI)."""
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
    U.custom("group8_window", 1, 520, 8, 1, 128, 200, 200, docs=(60, 400)),
    # no profiles, D 128, paired heads
    U.custom("no_profiles_pairs", 2, 300, 8, 2, 128, 0, 0, docs=(30, 250), pad=(0, 20)),
]

NAMES = ("dq", "dk", "dv", "dprofiles", "dsink")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from learned_relative_gqa_b200 import build
    build.build()


def check_full_bwd(x, with_dlse=False):
    out, lse = U.gpu_forward(x)
    dlse = None
    if with_dlse:
        g = torch.Generator(device="cuda").manual_seed(5)
        dlse = torch.randn(lse.shape, generator=g, device="cuda")
    grads = U.gpu_backward(x, out, lse, dlse)
    torch.cuda.synchronize()
    h = U.to_host(x)
    ref = U.oracle_backward(h, None if dlse is None else dlse.cpu().double().numpy())
    for n in NAMES:
        U.assert_grad_close(grads[n].cpu().numpy(), ref[n], n)


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_backward_small_shapes(w):
    check_full_bwd(W.make_inputs(w, "cuda", with_dout=True))


@pytest.mark.parametrize("w", SMALL[:4], ids=[w.name for w in SMALL[:4]])
def test_backward_small_shapes_with_lse_gradient(w):
    check_full_bwd(W.make_inputs(w, "cuda", with_dout=True), with_dlse=True)


def test_backward_pr1_ref_full():
    check_full_bwd(W.make_inputs(W.BY_NAME["pr1_ref"], "cuda", with_dout=True), with_dlse=True)


def test_backward_local_layer_full():
    check_full_bwd(W.make_inputs(W.BY_NAME["local"], "cuda", with_dout=True))


def test_backward_training_step_sampled():
    import oracle
    w = W.BY_NAME["train"]
    x = W.make_inputs(w, "cuda")
    out, lse = U.gpu_forward(x)
    grads = U.gpu_backward(x, out, lse)
    torch.cuda.synchronize()
    B, S, Hq, D = x["q"].shape
    Skv, Hkv = x["k"].shape[1], x["k"].shape[2]
    rows = U.sample_rows(x, 96)
    rng = np.random.default_rng(1)
    key_cols = [(b, j) for b in range(B) for j in (0, 1, S // 3, S - 1)]
    key_cols += [(int(rng.integers(B)), int(rng.integers(Skv))) for _ in range(4)]
    keys = np.array(sorted({(b * Skv + j) * Hkv + int(rng.integers(Hkv)) for b, j in key_cols}), dtype=np.int64)
    h = U.to_host(x)
    ref = oracle.backward_sampled(h["q"], h["k"], h["v"], h["profiles"], h["sink"], h["valid"], h["key_valid"],
                                  h["positions"], h["key_positions"], dout=h["dout"], rows=rows, keys=keys,
                                  window=h["window"], query_offset=h["query_offset"])
    R = x["profiles"].shape[3]
    dq = grads["dq"].cpu().numpy().reshape(-1, D)[rows]
    dsink = grads["dsink"].cpu().numpy().reshape(-1)[rows]
    # dprofiles rows are [b, h, i]: map (b, i, h) row ids
    bi, hh = rows // Hq, rows % Hq
    bb, ii = bi // S, bi % S
    prow = (bb * Hq + hh) * S + ii
    dprof = grads["dprofiles"].cpu().numpy().reshape(-1, R)[prow]
    U.assert_grad_close(dq, ref["dq"].reshape(-1, D)[rows], "dq")
    U.assert_grad_close(dsink, ref["dsink"].reshape(-1)[rows], "dsink")
    U.assert_grad_close(dprof, ref["dprofiles"].reshape(-1, R)[prow], "dprofiles")
    dk = grads["dk"].cpu().numpy().reshape(-1, D)[keys]
    dv = grads["dv"].cpu().numpy().reshape(-1, D)[keys]
    U.assert_grad_close(dk, ref["dk"].reshape(-1, D)[keys], "dk")
    U.assert_grad_close(dv, ref["dv"].reshape(-1, D)[keys], "dv")
    # properties of every element
    for n in NAMES:
        assert torch.isfinite(grads[n]).all(), n
    inval = ~x["valid"].bool()
    if inval.any():
        assert (grads["dq"][inval] == 0).all()


def test_backward_is_deterministic():
    x = W.make_inputs(U.custom("det", 1, 384, 8, 2, 128, 0, 128, docs=(50, 300)), "cuda", with_dout=True)
    out, lse = U.gpu_forward(x)
    a = U.gpu_backward(x, out, lse)
    b = U.gpu_backward(x, out, lse)
    for n in NAMES:
        assert torch.equal(a[n], b[n]), n


def test_forward_and_backward_replay_from_a_cuda_graph():
    """Forward + backward captured in a CUDA graph (the backward forks its dQ and
    zeroing work onto a second stream and joins it with events) replay to the same
    bits as the eager calls."""
    x = W.make_inputs(U.custom("graph", 2, 384, 8, 2, 128, 128, 128, docs=(50, 300), pad=(0, 30)), "cuda",
                      with_dout=True)
    out0, lse0 = U.gpu_forward(x)
    g0 = U.gpu_backward(x, out0, lse0)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):
            o, l = U.gpu_forward(x)
            U.gpu_backward(x, o, l)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out1, lse1 = U.gpu_forward(x)
        g1 = U.gpu_backward(x, out1, lse1)
    for t in (out1, lse1, *g1.values()):
        t.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out1, out0) and torch.equal(lse1, lse0)
    for n in NAMES:
        assert torch.equal(g1[n], g0[n]), n


def test_backward_with_a_running_maximum_that_grows_every_step():
    """The forward of test_forward_running_maximum_grows_every_step (O rescaled in every
    step) feeding the backward: probabilities recomputed from its log-sum-exp."""
    from tests.test_parity_fwd import ramp_profiles
    w = U.custom("growing_max", 1, 320, 4, 2, 128, 0, 320, docs=(150, 300))
    x = W.make_inputs(w, "cuda", with_dout=True)
    ramp_profiles(x, 0.25)
    check_full_bwd(x, with_dlse=True)
