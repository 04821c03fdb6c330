"""Device-side guards: bounded waits report instead of hanging, the device
error word reads clean after normal calls, and validate() rejects inputs that
break the preconditions."""
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


def test_bounded_wait_times_out_and_reports():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    st = binding.inkling_rel_attn_selftest_wait_timeout(2000, ws)   # 2 ms limit, nothing ever arrives
    assert st == binding.INKLING_ERR_TIMEOUT
    # the record is cleared once read
    assert binding.inkling_rel_attn_last_device_error(ws) == binding.INKLING_OK


def test_normal_calls_leave_no_device_error():
    x = W.make_inputs(U.custom("g", 1, 256, 4, 2, 128, 0, 64, docs=(40, 200)), "cuda", with_dout=True)
    dims = binding.make_dims(x["q"], x["k"], x["profiles"], 0)
    ws = binding.alloc_workspace(dims, True, "cuda")
    out, lse = binding.forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                               x["positions"], x["key_positions"], workspace=ws)
    assert binding.inkling_rel_attn_last_device_error(ws) == binding.INKLING_OK
    binding.backward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"], x["positions"],
                     x["key_positions"], out, lse, x["dout"], workspace=ws)
    assert binding.inkling_rel_attn_last_device_error(ws) == binding.INKLING_OK


def test_forward_abort_path_reports_a_timeout_and_the_context_survives():
    """With the pipeline waits limited to 1 ns, a CTA's first wait that does not
    succeed at once (its MMA issuer's wait for the Q tile) runs out: the CTA records
    the site, stops every role, drains its copies and products with the default limit
    and exits. The call reports the timeout; the same call with the default limit then
    completes and matches the oracle, so the context is intact."""
    x = W.make_inputs(U.custom("abort", 1, 256, 4, 2, 128, 0, 64, docs=(40, 200)), "cuda")
    dims = binding.make_dims(x["q"], x["k"], x["profiles"], 0)
    ws = binding.alloc_workspace(dims, False, "cuda")
    args = (x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"], x["positions"],
            x["key_positions"])
    binding.inkling_rel_attn_set_wait_timeout_ns(1)
    try:
        binding.forward(*args, workspace=ws)
        torch.cuda.synchronize()
        st = binding.inkling_rel_attn_last_device_error(ws)
    finally:
        binding.inkling_rel_attn_set_wait_timeout_ns(0)
    assert st == binding.INKLING_ERR_TIMEOUT
    out, lse = binding.forward(*args, workspace=ws)
    torch.cuda.synchronize()
    assert binding.inkling_rel_attn_last_device_error(ws) == binding.INKLING_OK
    o_ref, l_ref, _ = U.oracle_forward(U.to_host(x))
    U.assert_out_close(out.cpu().numpy(), o_ref)
    U.assert_lse_close(lse.cpu().numpy(), l_ref)


def _validate(x):
    dims = binding.make_dims(x["q"], x["k"], x["profiles"], x["window"], x["query_offset"])
    ws = binding.alloc_workspace(dims, False, "cuda")
    return binding.inkling_rel_attn_validate(dims, x["valid"], x["key_valid"], x["positions"], x["key_positions"], ws)


@pytest.mark.parametrize("name", ["pr1_ref", "local", "packed", "train"])
def test_validate_accepts_generated_workloads(name):
    assert _validate(W.make_inputs(W.BY_NAME[name], "cuda")) == binding.INKLING_OK


def test_validate_accepts_query_offset_slice():
    w = U.custom("cp", 2, 160, 4, 1, 128, 0, 96, docs=(30, 150), seq_k=384, query_offset=200)
    assert _validate(W.make_inputs(w, "cuda")) == binding.INKLING_OK


@pytest.mark.parametrize("break_it", ["position_jump", "negative_position", "hole_in_valid",
                                      "key_positions_disagree", "key_valid_disagrees"])
def test_validate_rejects_malformed(break_it):
    x = W.make_inputs(U.custom("m", 2, 256, 4, 2, 128, 0, 64, docs=(30, 120), pad=(5, 30)), "cuda")
    x["key_positions"] = x["key_positions"].clone()
    x["key_valid"] = x["key_valid"].clone()
    if break_it == "position_jump":
        x["positions"][0, 10] += 3
        x["key_positions"][0, 10] += 3
    elif break_it == "negative_position":
        x["positions"][1, 0] = -1
        x["key_positions"][1, 0] = -1
    elif break_it == "hole_in_valid":
        x["valid"][0, 50] = False
        x["key_valid"][0, 50] = False
    elif break_it == "key_positions_disagree":
        x["key_positions"][1, 77] += 1
    elif break_it == "key_valid_disagrees":
        x["key_valid"][0, 5] = False
    assert _validate(x) == binding.INKLING_ERR_MALFORMED_POSITIONS


def test_timing_hook_records_every_kernel():
    import ctypes
    x = W.make_inputs(U.custom("h", 1, 256, 4, 2, 128, 0, 64, docs=(40, 200)), "cuda", with_dout=True)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    arr = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in ev])
    binding.inkling_rel_attn_set_timing_events(arr, 3)
    try:
        U.gpu_forward(x)
    finally:
        binding.inkling_rel_attn_set_timing_events(None, 0)
    torch.cuda.synchronize()
    for k in range(3):
        assert ev[2 * k].elapsed_time(ev[2 * k + 1]) >= 0.0
