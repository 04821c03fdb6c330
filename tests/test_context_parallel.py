"""Context-parallel (sequence-sharded) attention: host-side orchestration on two
gloo ranks on the CPU, with the FP64 oracle as the per-rank attention, against
the unsharded oracle; and, on a GPU, the kernels' sharded results (local query
slices against the global keys, dK / dV summed over the slices) against the
unsharded kernels."""
import os
import socket

import numpy as np
import pytest
import torch

from learned_relative_gqa_b200 import workloads as W

WL = W.Workload("cp_small", 2, 96, 4, 2, 16, 40, 24, docs=(10, 50), pad=(0, 9), backward=True)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _dec(t):
    import oracle
    return oracle.decode_bf16(t.contiguous().view(torch.int16).numpy())


def _u8(t):
    return t.numpy().astype(np.uint8)


def _i32(t):
    return t.numpy().astype(np.int32)


def oracle_forward(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, *, window, query_offset):
    import oracle
    o, l, _ = oracle.forward(_dec(q), _dec(k), _dec(v), _dec(profiles), sink.double().numpy(), _u8(valid),
                             _u8(key_valid), _i32(positions), _i32(key_positions), window=window,
                             query_offset=query_offset)
    return torch.from_numpy(o), torch.from_numpy(l)


def oracle_backward(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout, dlse, *,
                    window, query_offset):
    import oracle
    g = oracle.backward(_dec(q), _dec(k), _dec(v), _dec(profiles), sink.double().numpy(), _u8(valid),
                        _u8(key_valid), _i32(positions), _i32(key_positions), dout=dout.double().numpy(),
                        dlse=None if dlse is None else dlse.double().numpy(), window=window,
                        query_offset=query_offset)
    return {n: torch.from_numpy(a) for n, a in g.items()}


def _slice_inputs(x, rank, world):
    S = x["q"].shape[1]
    n = S // world
    sl = slice(rank * n, (rank + 1) * n)
    loc = {}
    for name in ("q", "k", "v", "sink", "valid", "key_valid", "positions", "key_positions", "dout"):
        loc[name] = x[name][:, sl].contiguous()
    loc["profiles"] = x["profiles"][:, :, sl].contiguous()
    return loc, sl


def _rank_main(rank, world, port, result_dir):
    import torch.distributed as dist
    from learned_relative_gqa_b200 import context_parallel as cp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = W.make_inputs(WL, "cpu", with_dout=True)
        loc, sl = _slice_inputs(x, rank, world)
        out, lse = cp.forward(loc["q"], loc["k"], loc["v"], loc["profiles"], loc["sink"], loc["valid"],
                              loc["key_valid"], loc["positions"], loc["key_positions"], window=x["window"],
                              attn_forward=oracle_forward)
        g = cp.backward(loc["q"], loc["k"], loc["v"], loc["profiles"], loc["sink"], loc["valid"],
                        loc["key_valid"], loc["positions"], loc["key_positions"], out, lse, loc["dout"],
                        window=x["window"], attn_backward=oracle_backward)
        # the unsharded oracle, on every rank, for its own slice
        o_ref, l_ref = oracle_forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                                      x["positions"], x["key_positions"], window=x["window"], query_offset=0)
        g_ref = oracle_backward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                                x["positions"], x["key_positions"], o_ref, l_ref, x["dout"], None,
                                window=x["window"], query_offset=0)
        errs = {
            "out": float((out - o_ref[:, sl]).abs().max()),
            "lse": float((lse - l_ref[:, sl]).abs().max()),
            "dq": float((g["dq"] - g_ref["dq"][:, sl]).abs().max()),
            "dsink": float((g["dsink"] - g_ref["dsink"][:, sl]).abs().max()),
            "dprofiles": float((g["dprofiles"] - g_ref["dprofiles"][:, :, sl]).abs().max()),
            "dk": float((g["dk"] - g_ref["dk"][:, sl]).abs().max()),
            "dv": float((g["dv"] - g_ref["dv"][:, sl]).abs().max()),
            "dk_scale": float(g_ref["dk"].abs().max()),
        }
        torch.save(errs, os.path.join(result_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_context_parallel_two_gloo_ranks_match_the_unsharded_oracle(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        errs = torch.load(os.path.join(tmp_path, f"rank{r}.pt"))
        assert errs["dk_scale"] > 0
        for name, e in errs.items():
            if name != "dk_scale":
                assert e < 1e-9, f"rank {r} {name}: {e}"


def test_reduce_scatter_and_gather_single_rank_are_identity():
    import torch.distributed as dist
    from learned_relative_gqa_b200 import context_parallel as cp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        t = torch.arange(24, dtype=torch.float32).reshape(1, 6, 4)
        assert torch.equal(cp.gather_sequence(t), t)
        assert torch.equal(cp.reduce_scatter_sequence(t), t)
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_sharded_kernels_match_unsharded_kernels():
    """The context-parallel split on one GPU without collectives: each query slice
    against the global keys at its query_offset; dK / dV summed over the slices."""
    from learned_relative_gqa_b200 import binding
    w = W.Workload("cp_gpu", 2, 1024, 8, 2, 128, 256, 256, docs=(100, 700), pad=(0, 40), backward=True)
    x = W.make_inputs(w, "cuda", with_dout=True)
    full_out, full_lse = binding.forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"],
                                         x["key_valid"], x["positions"], x["key_positions"], window=x["window"])
    full_g = binding.backward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"],
                              x["positions"], x["key_positions"], full_out, full_lse, x["dout"], window=x["window"])
    world = 4
    dk = torch.zeros_like(full_g["dk"])
    dv = torch.zeros_like(full_g["dv"])
    for r in range(world):
        loc, sl = _slice_inputs(x, r, world)
        out, lse = binding.forward(loc["q"], x["k"], x["v"], loc["profiles"], loc["sink"], loc["valid"],
                                   x["key_valid"], loc["positions"], x["key_positions"], window=x["window"],
                                   query_offset=sl.start)
        g = binding.backward(loc["q"], x["k"], x["v"], loc["profiles"], loc["sink"], loc["valid"], x["key_valid"],
                             loc["positions"], x["key_positions"], out, lse, loc["dout"], window=x["window"],
                             query_offset=sl.start)
        torch.cuda.synchronize()
        torch.testing.assert_close(out, full_out[:, sl], rtol=0, atol=2e-5)
        torch.testing.assert_close(lse, full_lse[:, sl], rtol=0, atol=2e-5)
        torch.testing.assert_close(g["dq"], full_g["dq"][:, sl], rtol=0, atol=2e-4)
        torch.testing.assert_close(g["dsink"], full_g["dsink"][:, sl], rtol=0, atol=2e-5)
        torch.testing.assert_close(g["dprofiles"], full_g["dprofiles"][:, :, sl], rtol=0, atol=2e-5)
        dk += g["dk"]
        dv += g["dv"]
    scale = max(float(full_g["dk"].abs().max()), float(full_g["dv"].abs().max()))
    assert float((dk - full_g["dk"]).abs().max()) <= 1e-4 * scale
    assert float((dv - full_g["dv"]).abs().max()) <= 1e-4 * scale
