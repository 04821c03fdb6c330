"""CPU checks of the benchmark's host-side accounting: the allowed-element counts
behind the FLOP figures, the counts of elements that read a profile entry behind
the roofline bytes, the traffic lookup keyed by kernel source hashes, and the
reference arm's one JSON line under a two-rank launcher."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch

from learned_relative_gqa_b200 import workloads as W
from tests import dense_reference as ref

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

SHAPES = [
    W.Workload("c1", 2, 96, 4, 2, 16, 0, 24, docs=(10, 50), pad=(0, 9)),
    W.Workload("c2", 1, 130, 2, 1, 16, 20, 8, docs=(5, 60)),
    W.Workload("c3", 2, 80, 2, 2, 16, 0, 200, pad=(0, 30)),
    W.Workload("c4", 2, 64, 2, 1, 16, 0, 16, docs=(10, 30), seq_k=160, query_offset=70),
]


def dense_counts(x):
    m = ref.allowed_mask(x["valid"], x["key_valid"], x["positions"], x["key_positions"], window=x["window"],
                         query_offset=x["query_offset"], heads_q=x["q"].shape[2])
    S, Skv = x["q"].shape[1], x["k"].shape[1]
    dist = (torch.arange(S).view(S, 1) + x["query_offset"]) - torch.arange(Skv).view(1, Skv)
    R = x["profiles"].shape[3]
    return int(m.sum()), int((m & (dist < R)).sum())


@pytest.mark.parametrize("w", SHAPES, ids=[w.name for w in SHAPES])
def test_allowed_and_profile_reading_counts_match_a_dense_mask(w):
    x = W.make_inputs(w, "cpu")
    E_dense, Ep_dense = dense_counts(x)
    E = W.allowed_counts(w, x)
    assert E == E_dense
    assert bench.count_ep(x, E) == Ep_dense


def test_kernel_model_flops_are_the_metric_split():
    x = W.make_inputs(SHAPES[0], "cpu")
    E = W.allowed_counts(SHAPES[0], x)
    m = bench.kernel_model(x, E, bench.count_ep(x, E))
    D = x["q"].shape[3]
    assert m["fwd:attn_fwd"]["flops"] == 4.0 * D * E
    assert m["bwd:attn_bwd_dkdv"]["flops"] + m["bwd:attn_bwd_dq"]["flops"] == 14.0 * D * E
    assert all(v["bytes"] > 0 for v in m.values())


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    d = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    for k, v in d["kernels"].items():
        got = bench.ncu_traffic(k)
        if v["source_hash"] == bench.kernel_source_hash(k):
            assert got == v["bytes_per_launch_full_size"]
        else:
            assert got is None
    # a source file that differs from the one recorded makes the figure disappear
    k = "bwd:attn_bwd_dkdv"
    h = bench.kernel_source_hash(k, read=lambda name: b"changed " + name.encode())
    assert h != bench.kernel_source_hash(k)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_prints_one_line_under_two_ranks():
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_gpu_arm_refuses_a_world_size_other_than_gpus():
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--steps", "1", "--warmup", "1"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 2 and "WORLD_SIZE=3" in r.stderr


def test_gpu_arm_without_a_launcher_spawns_one_rank_per_gpu(monkeypatch):
    import bench
    calls = []
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: calls.append(cmd) or 0)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "2"])
    assert bench.spawn_ranks(4) == 0
    cmd = calls[0]
    assert cmd[1:3] == ["-m", "torch.distributed.run"] and "--nproc-per-node=4" in cmd
    assert "--master-addr=127.0.0.1" in cmd and cmd[-4:] == ["--gpus", "4", "--steps", "2"]
