"""Context-parallel (sequence-sharded) attention.

On the CPU: two gloo ranks run the host-side orchestration (an asynchronous
key all-gather overlapped with the local-diagonal block, the block of earlier
ranks' keys, the merge by log-sum-exp, the backward with the forward's gathered
keys and the dK / dV reduce-scatter) with the FP64 oracle as the per-rank
attention, against the unsharded oracle. On a GPU: four query slices emulated
one after another on one device (the gathered keys handed over directly), with
the library's kernels and merge, against the unsharded FP64 oracle at the
parity tolerances.
"""
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


def oracle_merge(out, lse, out_p, lse_p):
    """Merge of two results over disjoint key sets, in FP64 torch ops (test side)."""
    m = torch.maximum(lse, lse_p)
    safe = torch.where(torch.isinf(m), torch.zeros_like(m), m)
    wa, wb = torch.exp(lse - safe), torch.exp(lse_p - safe)
    s = wa + wb
    l = torch.where(s > 0, safe + torch.log(s), m)
    wa = torch.where(s > 0, wa / s, torch.zeros_like(s))
    wb = torch.where(s > 0, wb / s, torch.zeros_like(s))
    return out * wa[..., None] + out_p * wb[..., None], l


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
        out, lse, keys = cp.forward(loc["q"], loc["k"], loc["v"], loc["profiles"], loc["sink"], loc["valid"],
                                    loc["key_valid"], loc["positions"], loc["key_positions"], window=x["window"],
                                    attn_forward=oracle_forward, merge=oracle_merge, return_keys=True)
        g = cp.backward(loc["q"], loc["k"], loc["v"], loc["profiles"], loc["sink"], loc["valid"],
                        loc["key_valid"], loc["positions"], loc["key_positions"], out, lse, loc["dout"],
                        window=x["window"], attn_backward=oracle_backward, keys=keys)
        # the same backward with its own gather of the keys, and key_valid / key_positions
        # left to their defaults (valid / positions, as the single-GPU API)
        g2 = cp.backward(loc["q"], loc["k"], loc["v"], loc["profiles"], loc["sink"], loc["valid"], None,
                         loc["positions"], None, out, lse, loc["dout"], window=x["window"],
                         attn_backward=oracle_backward)
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
            "regather": max(float((g[n] - g2[n]).abs().max()) for n in g),
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
def test_four_slices_on_one_gpu_match_the_oracle():
    """The context-parallel forward and backward of four query slices, emulated one
    after another on one GPU: each slice's diagonal block, the block of the keys
    before it and their merge by the library, the backward against the global keys
    at the slice's query_offset; dK / dV summed over the slices. Compared with the
    unsharded FP64 oracle."""
    from learned_relative_gqa_b200 import context_parallel as cp
    from tests import parity_util as U
    w = W.Workload("cp_gpu", 2, 1024, 8, 2, 128, 256, 256, docs=(100, 700), pad=(0, 40), backward=True)
    x = W.make_inputs(w, "cuda", with_dout=True)
    h = U.to_host(x)
    o_ref, l_ref, _ = U.oracle_forward(h)
    g_ref = U.oracle_backward(h)
    world = 4
    full = cp.GatheredKeys(x["k"], x["v"], x["key_valid"], x["key_positions"])
    dk = torch.zeros_like(x["k"], dtype=torch.float32)
    dv = torch.zeros_like(dk)
    for r in range(world):
        loc, sl = _slice_inputs(x, r, world)
        out, lse, keys = cp.forward_shard(loc["q"], loc["k"], loc["v"], loc["profiles"], loc["sink"], loc["valid"],
                                          loc["key_valid"], loc["positions"], loc["key_positions"], rank=r,
                                          gathered=lambda: full, window=x["window"])
        from learned_relative_gqa_b200 import binding
        g = binding.backward(loc["q"], keys.k, keys.v, loc["profiles"], loc["sink"], loc["valid"], keys.key_valid,
                             loc["positions"], keys.key_positions, out, lse, loc["dout"], window=x["window"],
                             query_offset=sl.start)
        torch.cuda.synchronize()
        U.assert_out_close(out.cpu().numpy(), o_ref[:, sl], f"slice {r} out")
        U.assert_lse_close(lse.cpu().numpy(), l_ref[:, sl], f"slice {r} lse")
        U.assert_grad_close(g["dq"].cpu().numpy(), g_ref["dq"][:, sl], f"slice {r} dq")
        U.assert_grad_close(g["dsink"].cpu().numpy(), g_ref["dsink"][:, sl], f"slice {r} dsink")
        U.assert_grad_close(g["dprofiles"].cpu().numpy(), g_ref["dprofiles"][:, :, sl], f"slice {r} dprofiles")
        dk += g["dk"]
        dv += g["dv"]
    U.assert_grad_close(dk.cpu().numpy(), g_ref["dk"], "dk summed over slices")
    U.assert_grad_close(dv.cpu().numpy(), g_ref["dv"], "dv summed over slices")


@pytest.mark.gpu
def test_merge_of_two_key_halves_equals_the_whole():
    """inkling_rel_attn_merge: the keys split at a column into two disjoint sets (the
    sink counted in one), each half run by the kernels and merged by the library,
    give the unsplit FP64 oracle's result (each half rounds its probabilities to BF16
    against its own running maximum, so the merged result is not bit-equal to the
    kernels' unsplit one)."""
    from learned_relative_gqa_b200 import binding
    from tests import parity_util as U
    w = W.Workload("merge", 1, 512, 4, 2, 64, 0, 128, docs=(50, 400), backward=False)
    x = W.make_inputs(w, "cuda")
    o_ref, l_ref, _ = U.oracle_forward(U.to_host(x))
    cut = 200
    kv_a, kv_b = x["key_valid"].clone(), x["key_valid"].clone()
    kv_a[:, cut:] = 0
    kv_b[:, :cut] = 0
    o_a, l_a = binding.forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"], kv_a, x["positions"],
                               x["key_positions"])
    o_b, l_b = binding.forward(x["q"], x["k"], x["v"], x["profiles"], torch.full_like(x["sink"], float("-inf")),
                               x["valid"], kv_b, x["positions"], x["key_positions"])
    binding.inkling_rel_attn_merge(o_a, l_a, o_b, l_b)
    torch.cuda.synchronize()
    U.assert_out_close(o_a.cpu().numpy(), o_ref, "merged out")
    U.assert_lse_close(l_a.cpu().numpy(), l_ref, "merged lse")
    # rows whose keys all lie on one side of the cut are left as that side computed them
    kv = x["key_valid"].cpu().bool()
    assert bool(kv[:, :cut].any()) and bool(kv[:, cut:].any())
