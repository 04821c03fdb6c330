#!/usr/bin/env python
"""Benchmark of learned-relative GQA attention on B200.

A step is one pass of the whole hot path over one batch of synthetic input:
row bounds, the forward (QK^T, relative-profile gather, masked online softmax
with the sink, PV, epilogue) and the backward (preprocessing, dK/dV/dprofiles,
dQ) of the ``train`` workload (B2 S8192 Hq32 Hkv4 D128, window 1024, R 1024,
packed documents; the only workload with a backward). The metric counts only
allowed (unmasked) score elements E: 4*D*E forward + 10*D*E backward FLOPs.
The forward of the ``long`` workload (S 32768, R 4096, full causal) is timed
as well and reported under ``long_fwd``, and one forward + backward of the
generic FlexAttention variant on the packed-documents shape (EOS-delimited
documents, per-head sinks, [B, H, S, D] tensors) under ``flex_step``, and
L2Clip forward + backward on q of the training shape under ``l2clip``.

python bench.py --gpus N --steps K --warmup W [--impl reference]
Under torchrun each rank runs its own batch (weak scaling, no data-path
collective); the timed region is bracketed by a barrier and synchronize and
the max over ranks is reported. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "fwd/bwd rel-GQA attention TFLOP/s (unmasked FLOPs), % of B200 BF16 peak"
FWD_KERNELS = ["key_span", "row_bounds", "attn_fwd"]
BWD_KERNELS = ["key_span", "row_bounds", "bwd_prep", "dprof_zero", "attn_bwd_dkdv", "attn_bwd_dq"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# source files each kernel is built from (its own translation unit and the headers it includes)
KERNEL_SOURCES = {
    "fwd:attn_fwd": ["fwd.cu", "common.cuh", "launch.h", "ptx.cuh"],
    "bwd:attn_bwd_dkdv": ["bwd.cu", "common.cuh", "launch.h", "ptx.cuh"],
    "bwd:attn_bwd_dq": ["bwd.cu", "common.cuh", "launch.h", "ptx.cuh"],
    "bwd:bwd_prep": ["prep_kernels.cu", "common.cuh", "launch.h", "ptx.cuh"],
    "bwd:dprof_zero": ["prep_kernels.cu", "common.cuh", "launch.h", "ptx.cuh"],
}


def kernel_source_hash(kernel: str, read=None) -> str:
    """sha256 (first 16 hex digits) over the source files of `kernel`. `read(name)` returns a
    file's bytes (default: the working tree)."""
    csrc = os.path.join(ROOT, "learned_relative_gqa_b200", "csrc")
    if read is None:
        def read(name):
            with open(os.path.join(csrc, name), "rb") as f:
                return f.read()
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[kernel]):
        h.update(name.encode() + read(name))
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if it was
    taken on the current sources of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    with open(path) as f:
        d = json.load(f)
    k = d.get("kernels", {}).get(kernel)
    if k is None or k.get("source_hash") != kernel_source_hash(kernel):
        return None
    return k.get("bytes_per_launch_full_size")


class ClockSampler:
    """SM clock, power and clock-event reasons sampled every few milliseconds during the
    timed region, through NVML from a background thread (the timed loop spends its time
    in CUDA synchronisation, which releases the GIL). Falls back to ``nvidia-smi -lms``
    when NVML is unavailable. Samples are also written to ``path`` as CSV."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, device_index: int, path: str, period_s: float = 0.004):
        import threading
        self.path, self.period = path, period_s
        os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
        self.rows, self.proc, self.thread = [], None, None
        self.stop_evt = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.nvml, self.handle = pynvml, pynvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.sample()  # one sample before the timed region starts
            self.rows.clear()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
        except Exception:
            self.nvml = None
            q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            try:
                self.f = open(path, "w")
                self.proc = subprocess.Popen(["nvidia-smi", f"--id={device_index}", f"--query-gpu={q}",
                                              "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                             stderr=subprocess.DEVNULL)
            except Exception:
                self.proc = None

    def sample(self):
        nv = self.nvml
        sm = float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
        try:
            mask = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
        except Exception:
            mask = int(nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle))
        power = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
        self.rows.append((time.time(), sm, self.max_mhz, power, mask))

    def _loop(self):
        while not self.stop_evt.is_set():
            try:
                self.sample()
            except Exception:
                return
            time.sleep(self.period)

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            try:
                self.sample()  # the state right at the end of the timed region
            except Exception:
                pass
            with open(self.path, "w") as f:
                f.write("time,sm_mhz,sm_max_mhz,power_w,reasons_mask\n")
                for r in self.rows:
                    f.write(f"{r[0]:.4f},{r[1]:.0f},{r[2]:.0f},{r[3]:.1f},{r[4]:#x}\n")
            if not self.rows:
                return None
            sm = sorted(r[1] for r in self.rows)
            reasons = sorted({name for r in self.rows for bit, name in self.REASONS.items() if r[4] & bit})
            return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(self.rows), "source": "nvml"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return None
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        mx = max((float(r[2]) for r in rows if r[2].replace(".", "").isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower().startswith("active")})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "source": "nvidia-smi"}


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_threads() -> int:
    """Give the oracle every core this process may use (a launcher such as torchrun sets
    OMP_NUM_THREADS=1 per rank) and return the thread count it then runs with."""
    import oracle
    return oracle.set_threads(cpu_cores())


# ---------------------------------------------------------------------------
# oracle sample (CPU baseline / reference arm)
# ---------------------------------------------------------------------------
def crop_inputs(x, s_sub: int, group: int = 0):
    """Batch 0, the query heads of one KV group, the first s_sub tokens."""
    Hq, Hkv = x["q"].shape[2], x["k"].shape[2]
    G = Hq // Hkv
    hs = slice(group * G, (group + 1) * G)
    gs = slice(group, group + 1)
    c = {
        "q": x["q"][:1, :s_sub, hs].contiguous(), "k": x["k"][:1, :s_sub, gs].contiguous(),
        "v": x["v"][:1, :s_sub, gs].contiguous(), "profiles": x["profiles"][:1, hs, :s_sub].contiguous(),
        "sink": x["sink"][:1, :s_sub, hs].contiguous(), "valid": x["valid"][:1, :s_sub].contiguous(),
        "key_valid": x["key_valid"][:1, :s_sub].contiguous(), "positions": x["positions"][:1, :s_sub].contiguous(),
        "key_positions": x["key_positions"][:1, :s_sub].contiguous(),
        "dout": x["dout"][:1, :s_sub, hs].contiguous(), "window": x["window"], "query_offset": 0,
        "rel_extent": x["rel_extent"],
    }
    return c


def oracle_sample_step(hc):
    import oracle
    o, l, _ = oracle.forward(hc["q"], hc["k"], hc["v"], hc["profiles"], hc["sink"], hc["valid"], hc["key_valid"],
                             hc["positions"], hc["key_positions"], window=hc["window"])
    oracle.backward(hc["q"], hc["k"], hc["v"], hc["profiles"], hc["sink"], hc["valid"], hc["key_valid"],
                    hc["positions"], hc["key_positions"], dout=hc["dout"], window=hc["window"])
    return o, l


def host_sample(x, s_sub):
    import numpy as np
    import oracle
    from learned_relative_gqa_b200 import workloads
    c = crop_inputs(x, s_sub)
    hc = {n: oracle.decode_bf16(c[n].cpu().view(torch.int16).numpy()) for n in ("q", "k", "v", "profiles")}
    hc["sink"] = c["sink"].cpu().double().numpy()
    hc["dout"] = c["dout"].cpu().double().numpy()
    for n in ("valid", "key_valid"):
        hc[n] = c[n].cpu().numpy().astype(np.uint8)
    for n in ("positions", "key_positions"):
        hc[n] = c[n].cpu().numpy().astype(np.int32)
    hc["window"] = c["window"]
    w = workloads.Workload("sample", 1, s_sub, c["q"].shape[2], 1, c["q"].shape[3], c["window"], c["rel_extent"])
    E = workloads.allowed_counts(w, c)
    return hc, E


def calibrate_sample(x, target_s: float = 8.0, max_s: float = 20.0):
    """Largest prefix (power-of-two tokens) whose oracle fwd+bwd takes about target_s."""
    S = x["q"].shape[1]
    s_sub = 256
    while True:
        hc, E = host_sample(x, s_sub)
        t0 = time.perf_counter()
        oracle_sample_step(hc)
        dt = time.perf_counter() - t0
        if dt * 4 > max_s or s_sub * 2 > S or dt > target_s:
            return s_sub, hc, E, dt
        s_sub *= 2


def cpu_baseline(x, D, budget_s=20.0):
    threads = oracle_threads()
    s_sub, hc, E, dt = calibrate_sample(x, max_s=budget_s)
    if dt < 5.0:  # re-time on the chosen sample
        reps = max(1, int(5.0 / max(dt, 1e-3)))
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle_sample_step(hc)
        dt = (time.perf_counter() - t0) / reps
    flops = 14.0 * D * E
    G = hc["q"].shape[2]
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": (f"FP64 oracle forward+backward on batch 0, one KV group ({G} query heads), first {s_sub} "
                       f"tokens of the same workload: E={E} allowed elements, {dt:.2f} s per step")}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
class Buffers:
    def __init__(self, x, backward: bool):
        from learned_relative_gqa_b200 import binding
        self.x = x
        dev = x["q"].device
        self.dims = binding.make_dims(x["q"], x["k"], x["profiles"], x["window"], x["query_offset"])
        f32 = dict(dtype=torch.float32, device=dev)
        self.out = torch.empty(x["q"].shape, **f32)
        self.lse = torch.empty(x["q"].shape[:3], **f32)
        self.ws = binding.alloc_workspace(self.dims, backward, dev)
        if backward:
            self.dq = torch.empty(x["q"].shape, **f32)
            self.dk = torch.empty(x["k"].shape, **f32)
            self.dv = torch.empty(x["v"].shape, **f32)
            self.dprof = torch.empty(x["profiles"].shape, **f32)
            self.dsink = torch.empty(x["sink"].shape, **f32)

    def fwd(self):
        from learned_relative_gqa_b200 import binding
        x = self.x
        binding.inkling_rel_attn_fwd(self.dims, x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"],
                                     x["key_valid"], x["positions"], x["key_positions"], self.out, self.lse, self.ws)

    def bwd(self):
        from learned_relative_gqa_b200 import binding
        x = self.x
        binding.inkling_rel_attn_bwd(self.dims, x["q"], x["k"], x["v"], x["profiles"], x["sink"], x["valid"],
                                     x["key_valid"], x["positions"], x["key_positions"], self.out, self.lse,
                                     x["dout"], None, self.dq, self.dk, self.dv, self.dprof, self.dsink, self.ws)


def timed(fn, steps, sync_all):
    sync_all()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        fn()
    end.record()
    sync_all()
    return start.elapsed_time(end)


def per_kernel_times(buf: Buffers, steps: int, backward: bool):
    """Average duration (ms) of each library kernel, from the timing-event hook."""
    from learned_relative_gqa_b200 import binding
    names_f = FWD_KERNELS
    names_b = BWD_KERNELS if backward else []
    nf, nb = len(names_f), len(names_b)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * (nf + nb))] for _ in range(steps)]
    for e in ev:
        for x in e:
            x.record()  # torch creates the CUDA event lazily, on first record
    torch.cuda.synchronize()
    arrays = []
    for e in ev:
        fa = (ctypes.c_void_p * (2 * nf))(*[ctypes.c_void_p(x.cuda_event) for x in e[:2 * nf]])
        ba = (ctypes.c_void_p * (2 * nb))(*[ctypes.c_void_p(x.cuda_event) for x in e[2 * nf:]]) if nb else None
        arrays.append((fa, ba))
    for fa, ba in arrays:
        binding.inkling_rel_attn_set_timing_events(fa, nf)
        buf.fwd()
        if backward:
            binding.inkling_rel_attn_set_timing_events(ba, nb)
            buf.bwd()
    binding.inkling_rel_attn_set_timing_events(None, 0)
    torch.cuda.synchronize()
    acc = {}
    for e in ev:
        for k, n in enumerate(names_f):
            acc.setdefault("fwd:" + n, []).append(e[2 * k].elapsed_time(e[2 * k + 1]))
        for k, n in enumerate(names_b):
            acc.setdefault("bwd:" + n, []).append(e[2 * nf + 2 * k].elapsed_time(e[2 * nf + 2 * k + 1]))
    return {k: sum(v) / len(v) for k, v in acc.items()}


def kernel_model(x, E, Ep):
    """Algorithmic FLOPs and bytes per launch of the attention kernels.

    E  = allowed (row, key, head) elements; Ep = those with distance < R.
    """
    B, S, Hq, D = x["q"].shape
    Skv, Hkv = x["k"].shape[1], x["k"].shape[2]
    R = x["profiles"].shape[3]
    q_b = B * S * Hq * D * 2
    kv_b = 2 * B * Skv * Hkv * D * 2
    rows = B * S * Hq
    return {
        "fwd:attn_fwd": dict(flops=4.0 * D * E, bytes=q_b + kv_b + 2.0 * Ep + rows * (4 * D + 4) + rows * 4),
        "bwd:attn_bwd_dkdv": dict(flops=8.0 * D * E,
                                  bytes=q_b * 2 + kv_b + 2.0 * Ep + 4.0 * Ep + B * Skv * Hkv * D * 8 + rows * 8),
        "bwd:attn_bwd_dq": dict(flops=6.0 * D * E, bytes=q_b * 2 + kv_b + 2.0 * Ep + rows * (4 * D + 8)),
        "bwd:bwd_prep": dict(flops=2.0 * rows * D, bytes=rows * (8 * D + 2 * D + 20)),
        "bwd:dprof_zero": dict(flops=0.0, bytes=4.0 * (B * Hq * S * R - Ep) + rows * 8),
    }


def count_ep(x, E):
    """Allowed elements whose distance is < R (the ones that read / write a profile entry)."""
    W, R = x["window"], x["profiles"].shape[3]
    if W > 0 and W <= R:
        return E
    valid = x["valid"].cpu()
    kvalid = x["key_valid"].cpu()
    pos = x["positions"].cpu().to(torch.int64)
    B, S = valid.shape
    ig = torch.arange(S, dtype=torch.int64) + x["query_offset"]
    total = 0
    for b in range(B):
        idx = torch.nonzero(kvalid[b]).flatten()
        if idx.numel() == 0:
            continue
        lo = torch.maximum(ig - pos[b], torch.full_like(ig, int(idx[0])))
        if W > 0:
            lo = torch.maximum(lo, ig - W + 1)
        lo = torch.maximum(lo, ig - R + 1)
        hi = torch.minimum(ig, torch.full_like(ig, int(idx[-1])))
        total += int(((hi - lo + 1).clamp(min=0) * valid[b].to(torch.int64)).sum())
    return total * x["q"].shape[2]


def e2e_run(x, steps, backward):
    """Same step through the public API from pinned host buffers: H2D of the inputs,
    the library calls, D2H of every result, each step. Consecutive steps overlap on
    three streams (copy-in, kernels, copy-out) with two device buffer sets, so the
    inputs of step k+1 travel in while step k computes and the results of step k-1
    travel out (PCIe is full duplex); every step still moves all of its own bytes."""
    from learned_relative_gqa_b200 import binding
    names_in = ["q", "k", "v", "profiles", "sink", "valid", "key_valid", "positions", "key_positions"]
    if backward:
        names_in.append("dout")
    host = {n: x[n].cpu().pin_memory() for n in names_in}
    slots = []
    for _ in range(2):
        dev = {n: torch.empty_like(x[n]) for n in names_in}
        for n in ("window", "query_offset"):
            dev[n] = x[n]
        buf = Buffers(dev, backward)
        outs = [buf.out, buf.lse] + ([buf.dq, buf.dk, buf.dv, buf.dprof, buf.dsink] if backward else [])
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        slots.append((dev, buf, outs, host_out))
    h2d = sum(host[n].numel() * host[n].element_size() for n in names_in)
    d2h = sum(t.numel() * t.element_size() for t in slots[0][2])
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def run(nsteps):
        comp_done = [None] * nsteps
        out_done = [None] * nsteps
        for k in range(nsteps):
            dev, buf, outs, host_out = slots[k % 2]
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(comp_done[k - 2])   # the slot's inputs were read by step k-2
                for n in names_in:
                    dev[n].copy_(host[n], non_blocking=True)
                in_done = torch.cuda.Event()
                in_done.record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(in_done)
                if k >= 2:
                    s_comp.wait_event(out_done[k - 2])  # the slot's results of step k-2 are out
                buf.fwd()
                if backward:
                    buf.bwd()
                comp_done[k] = torch.cuda.Event()
                comp_done[k].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[k])
                for t, hb in zip(outs, host_out):
                    hb.copy_(t, non_blocking=True)
                out_done[k] = torch.cuda.Event()
                out_done[k].record(s_out)

    run(2)  # warm-up of both slots
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    run(steps)
    end.record(s_out)  # after the last copy-out, which follows every earlier operation
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    del binding
    return ms / steps, h2d, d2h


def spawn_ranks(n: int) -> int:
    """Re-runs this command under torch.distributed.run with n ranks on this node."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="train")
    ap.add_argument("--seq", type=int, default=0,
                    help="override the workload's sequence length (smaller cases for profiling)")
    ap.add_argument("--long-steps", type=int, default=3, help="forward steps of the long workload (0 = skip)")
    ap.add_argument("--flex-steps", type=int, default=3,
                    help="forward + backward steps of the generic FlexAttention variant (0 = skip)")
    ap.add_argument("--l2clip-steps", type=int, default=5, help="L2Clip forward + backward steps (0 = skip)")
    ap.add_argument("--qclip-steps", type=int, default=-1,
                    help="steps of the workload with the L2Clip of q fused in, and with it separate (-1: as l2clip)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-csv-dir", default="/tmp",
                    help="directory for the CSV of the SM clock samples taken during the timed regions")
    ap.add_argument("--e2e-steps", type=int, default=3)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "ours" and world != args.gpus:
        if "WORLD_SIZE" not in os.environ and args.gpus > 1:
            # not started by a launcher: start one rank per GPU on this node and pass
            # their exit status through (rank 0 prints the JSON line)
            sys.exit(spawn_ranks(args.gpus))
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU", file=sys.stderr)
        sys.exit(2)
    from learned_relative_gqa_b200 import workloads
    import dataclasses
    w = workloads.BY_NAME[args.workload]
    if args.seq > 0:
        w = dataclasses.replace(w, seq=args.seq)
    backward = w.backward
    if args.impl == "reference":
        # the oracle on the host cores; under torchrun only rank 0 works
        if rank == 0:
            run_reference(args, w, backward)
        return
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device(f"cuda:{local}"))
    device = torch.device(f"cuda:{local}")
    torch.cuda.set_device(device)

    def sync_all():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
            torch.cuda.synchronize()

    from learned_relative_gqa_b200 import binding, build
    build.build()
    binding.load()
    x = workloads.make_inputs(w, device, seed=workloads.seed_of(workloads.BY_NAME[args.workload]) + 7919 * rank)
    D = w.head_dim
    E = workloads.allowed_counts(w, x)
    Ep = count_ep(x, E)
    flops_step = (14.0 if backward else 4.0) * D * E
    buf = Buffers(x, backward)

    def step():
        buf.fwd()
        if backward:
            buf.bwd()

    for _ in range(args.warmup):
        step()
    sync_all()
    sampler = ClockSampler(local, os.path.join(args.clock_csv_dir, f"clocks_rank{rank}.csv"))
    ms = timed(step, args.steps, sync_all)
    clocks = sampler.stop()
    ms_t = torch.tensor([ms], device=device, dtype=torch.float64)
    if dist is not None:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    ms_step = ms_max / args.steps
    # every rank draws its own documents, so the job's FLOPs are the sum over ranks
    fl_t = torch.tensor([flops_step], device=device, dtype=torch.float64)
    if dist is not None:
        dist.all_reduce(fl_t, op=dist.ReduceOp.SUM)
    flops_job = float(fl_t.item())
    value = flops_job / (ms_step * 1e-3) / 1e12

    # per-kernel durations (events recorded on the launch stream around each kernel)
    kt = per_kernel_times(buf, args.steps, backward)
    gpu_launches = args.steps * (len(FWD_KERNELS) + (len(BWD_KERNELS) if backward else 0))
    if backward and x["profiles"].shape[3] == 0:
        gpu_launches -= args.steps
    peaks, peak_src = load_peaks()
    model = kernel_model(x, E, Ep)
    att = {k: v for k, v in kt.items() if k in model}
    dom = max(att, key=att.get)
    m = model[dom]
    t_s = att[dom] * 1e-3
    t_tc = m["flops"] / (peaks["bf16_tflops"] * 1e12)
    t_hbm = m["bytes"] / (peaks["hbm_gbs"] * 1e9)
    if t_tc >= t_hbm:
        roof = {"bound": "tensor", "achieved": m["flops"] / t_s / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": m["bytes"] / t_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["traffic"] = ncu_traffic(dom)
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json burst figures)" if peak_src == "measured" else "fallback"
    kernels = {k: {"ms": round(v, 4), "share": round(v / sum(kt.values()), 4)} for k, v in kt.items()}
    for k in kernels:
        if k in model:
            mm = model[k]
            kernels[k]["tflops"] = round(mm["flops"] / (kt[k] * 1e-3) / 1e12, 1)
            kernels[k]["gbs"] = round(mm["bytes"] / (kt[k] * 1e-3) / 1e9, 1)

    # end to end through host buffers
    e2e = None
    if args.e2e_steps > 0:
        e_ms, h2d, d2h = e2e_run(x, args.e2e_steps, backward)
        e_t = torch.tensor([e_ms], device=device, dtype=torch.float64)
        if dist is not None:
            dist.all_reduce(e_t, op=dist.ReduceOp.MAX)
        e2e = {"value": flops_job / (float(e_t.item()) * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(float(e_t.item()), 3),
               "overlap": "copy-in, kernels and copy-out of consecutive steps on three streams, two buffer sets"}

    # the long-context forward (spec forward target at S = 32768)
    long_fwd = None
    if args.long_steps > 0 and rank == 0 and args.workload != "long":
        del buf
        torch.cuda.empty_cache()
        wl = workloads.BY_NAME["long"]
        xl = workloads.make_inputs(wl, device)
        El = workloads.allowed_counts(wl, xl)
        bl = Buffers(xl, False)
        for _ in range(2):
            bl.fwd()
        torch.cuda.synchronize()
        sampler_l = ClockSampler(local, os.path.join(args.clock_csv_dir, f"clocks_long_rank{rank}.csv"))
        ms_l = timed(bl.fwd, args.long_steps, torch.cuda.synchronize) / args.long_steps
        clocks_l = sampler_l.stop()
        tfl = 4.0 * wl.head_dim * El / (ms_l * 1e-3) / 1e12
        long_fwd = {"workload": "long: B1 S32768 Hq32 Hkv8 D128 R4096 full causal", "ms": round(ms_l, 3),
                    "allowed_elements": El, "tflops": round(tfl, 1),
                    "pct_of_bf16_peak": round(100 * tfl / peaks["bf16_tflops"], 1), "clocks": clocks_l}
        del bl, xl
        torch.cuda.empty_cache()

    # the generic FlexAttention variant (same kernels, [B, H, S, D], BF16 output)
    flex_step = None
    if args.flex_steps > 0 and rank == 0:
        flex_step = flex_run(args.flex_steps, device, peaks)

    l2c = None
    if args.l2clip_steps > 0 and rank == 0:
        l2c = l2clip_run(args.l2clip_steps, device, peaks)
    qclip_steps = args.l2clip_steps if args.qclip_steps < 0 else args.qclip_steps
    if qclip_steps > 0 and rank == 0 and backward:
        torch.cuda.empty_cache()
        fused = qclip_run(qclip_steps, device, peaks, w)
        l2c = dict(l2c or {}, fused_step=fused)

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x, D)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": run_config(w, x, E, flops_step, world),
            "pct_of_bf16_peak": round(100 * value / world / peaks["bf16_tflops"], 2),
            "roofline": roof, "kernels": kernels, "gpu_launches": gpu_launches,
            "e2e": e2e, "cpu_baseline": cpu, "clocks": clocks, "long_fwd": long_fwd, "flex_step": flex_step,
            "l2clip": l2c,
        }
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def flex_run(steps, device, peaks):
    """Forward + backward of the generic variant on ``flex_packed`` through its C ABI,
    preallocated outputs and workspaces; inputs (q, k, v, dout, out: 0.54 GB) exceed L2."""
    from learned_relative_gqa_b200 import binding, workloads
    wf = workloads.FLEX_BY_NAME["flex_packed"]
    xf = workloads.make_flex_inputs(wf, device)
    E = workloads.flex_allowed_counts(wf, xf)
    kw = dict(mask_type=wf.mask_type, eos_id=wf.eos_id, fixed_block_size=wf.fixed_block_size,
              sliding_window=wf.sliding_window, scale=wf.scale, enable_gqa=wf.heads_q != wf.heads_kv)
    dims = binding.make_flex_dims(xf["q"], xf["k"], **kw)
    wsf = torch.empty(binding.inkling_flex_attn_workspace_size(dims, False), dtype=torch.uint8, device=device)
    wsb = torch.empty(binding.inkling_flex_attn_workspace_size(dims, True), dtype=torch.uint8, device=device)
    out = torch.empty(xf["q"].shape, dtype=torch.bfloat16, device=device)
    lse = torch.empty(xf["q"].shape[:3], dtype=torch.float32, device=device)
    f32 = dict(dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty(xf["q"].shape, **f32), torch.empty(xf["k"].shape, **f32), torch.empty(xf["v"].shape, **f32)
    dsw = torch.empty(xf["sink_weights"].shape, **f32)

    def fwd():
        binding.inkling_flex_attn_fwd(dims, xf["q"], xf["k"], xf["v"], xf["sink_weights"], xf["tokens"], out, lse, wsf)

    def bwd():
        binding.inkling_flex_attn_bwd(dims, xf["q"], xf["k"], xf["v"], xf["sink_weights"], xf["tokens"], out, lse,
                                      xf["dout"], dq, dk, dv, dsw, wsb)

    for _ in range(3):
        fwd()
        bwd()
    ms_f = timed(fwd, steps, torch.cuda.synchronize) / steps
    ms_b = timed(bwd, steps, torch.cuda.synchronize) / steps
    D = wf.head_dim
    tf_f = 4.0 * D * E / (ms_f * 1e-3) / 1e12
    tf_b = 10.0 * D * E / (ms_b * 1e-3) / 1e12
    tf = 14.0 * D * E / ((ms_f + ms_b) * 1e-3) / 1e12
    return {"workload": (f"flex_packed: B{wf.batch} S{wf.seq} Hq{wf.heads_q} Hkv{wf.heads_kv} D{D} "
                         f"{wf.mask_type} docs{wf.docs} sink_weights[Hq], [B,H,S,D], BF16 out"),
            "allowed_elements": E, "fwd_ms": round(ms_f, 3), "bwd_ms": round(ms_b, 3),
            "fwd_tflops": round(tf_f, 1), "bwd_tflops": round(tf_b, 1), "tflops": round(tf, 1),
            "pct_of_bf16_peak": round(100 * tf / peaks["bf16_tflops"], 1)}


def l2clip_run(steps, device, peaks):
    """L2Clip forward and backward (learned scales and length scaling on) on q of the
    training shape, B2 S8192 Hq32 D128: 134 MB of BF16 x; both passes are HBM streams
    (4 and 10 bytes per element), each larger than L2."""
    from learned_relative_gqa_b200 import binding
    B, S, H, D = 2, 8192, 32, 128
    g = torch.Generator(device)
    g.manual_seed(7)
    x = torch.randn(B, S, H, D, generator=g, device=device).to(torch.bfloat16)
    scale = 0.5 + torch.rand(H, D, generator=g, device=device)
    tau = 0.5 + torch.rand(B, S, generator=g, device=device)
    dy = torch.randn(B, S, H, D, generator=g, device=device)
    dims = binding.make_l2clip_dims(x, 9.0)
    y = torch.empty_like(x)
    dx = torch.empty(x.shape, dtype=torch.float32, device=device)
    dscale = torch.empty(H, D, dtype=torch.float32, device=device)
    dtau = torch.empty(B, S, dtype=torch.float32, device=device)
    ws = torch.empty(binding.inkling_l2clip_workspace_size(dims), dtype=torch.uint8, device=device)

    def fwd():
        binding.inkling_l2clip_fwd(dims, x, scale, tau, y)

    def bwd():
        binding.inkling_l2clip_bwd(dims, x, scale, tau, dy, dx, dscale, dtau, ws)

    for _ in range(3):
        fwd()
        bwd()
    ms_f = timed(fwd, steps, torch.cuda.synchronize) / steps
    ms_b = timed(bwd, steps, torch.cuda.synchronize) / steps
    n = B * S * H * D
    bf, bb = 4.0 * n, 10.0 * n
    return {"workload": f"L2Clip on q: B{B} S{S} H{H} D{D}, learned scales, tau, threshold 9",
            "fwd_ms": round(ms_f, 4), "bwd_ms": round(ms_b, 4),
            "fwd_gbs": round(bf / (ms_f * 1e-3) / 1e9, 1), "bwd_gbs": round(bb / (ms_b * 1e-3) / 1e9, 1),
            "fwd_frac_of_hbm": round(bf / (ms_f * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
            "bwd_frac_of_hbm": round(bb / (ms_b * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}


def qclip_run(steps, device, peaks, w):
    """The step of workload w with the L2Clip of q (learned scales, tau, threshold 9) fused
    into the attention kernels (inkling_rel_attn_fwd_qclip / _bwd_qclip), against the same
    step with the standalone L2Clip passes around the unfused attention; same inputs."""
    from learned_relative_gqa_b200 import binding, workloads
    x = workloads.make_inputs(w, device)
    B, S, Hq, D = x["q"].shape
    g = torch.Generator(device)
    g.manual_seed(11)
    xq = (x["q"].float() * (0.2 + 1.6 * torch.rand(B, S, Hq, 1, generator=g, device=device))).to(torch.bfloat16)
    scale = 0.5 + torch.rand(Hq, D, generator=g, device=device)
    tau = 0.5 + 1.5 * torch.rand(B, S, generator=g, device=device)
    thr = 9.0
    E = workloads.allowed_counts(w, x)
    dims = binding.make_dims(xq, x["k"], x["profiles"], x["window"], x["query_offset"])
    ldims = binding.make_l2clip_dims(xq, thr)
    f32 = dict(dtype=torch.float32, device=device)
    out, lse = torch.empty(xq.shape, **f32), torch.empty(xq.shape[:3], **f32)
    qc = torch.empty_like(xq)
    dx, dk, dv = torch.empty(xq.shape, **f32), torch.empty(x["k"].shape, **f32), torch.empty(x["v"].shape, **f32)
    dprof, dsink = torch.empty(x["profiles"].shape, **f32), torch.empty(x["sink"].shape, **f32)
    dscale, dtau, dq = torch.empty(Hq, D, **f32), torch.empty(B, S, **f32), torch.empty(xq.shape, **f32)
    lib = binding.load()
    ws = torch.empty(int(lib.inkling_rel_attn_qclip_workspace_size(ctypes.byref(dims), 1)), dtype=torch.uint8,
                     device=device)
    lws = torch.empty(binding.inkling_l2clip_workspace_size(ldims), dtype=torch.uint8, device=device)
    a = (x["k"], x["v"], x["profiles"], x["sink"], x["valid"], x["key_valid"], x["positions"], x["key_positions"])
    st = binding._stream(None)

    def fused():
        p = binding._p
        binding._check(lib.inkling_rel_attn_fwd_qclip(
            ctypes.byref(dims), thr, p(scale), p(tau), p(xq), *[p(t) for t in a[:4]], p(binding._u8(a[4])),
            p(binding._u8(a[5])), p(a[6]), p(a[7]), p(qc), p(out), p(lse), p(ws), ws.numel(), st), "fwd_qclip")
        binding._check(lib.inkling_rel_attn_bwd_qclip(
            ctypes.byref(dims), thr, p(scale), p(tau), p(xq), p(qc), *[p(t) for t in a[:4]], p(binding._u8(a[4])),
            p(binding._u8(a[5])), p(a[6]), p(a[7]), p(out), p(lse), p(x["dout"]), None, p(dx), p(dk), p(dv),
            p(dprof), p(dsink), p(dscale), p(dtau), p(ws), ws.numel(), st), "bwd_qclip")

    def separate():
        binding.inkling_l2clip_fwd(ldims, xq, scale, tau, qc)
        binding.inkling_rel_attn_fwd(dims, qc, *a, out, lse, ws)
        binding.inkling_rel_attn_bwd(dims, qc, *a, out, lse, x["dout"], None, dq, dk, dv, dprof, dsink, ws)
        binding.inkling_l2clip_bwd(ldims, xq, scale, tau, dq, dx, dscale, dtau, lws)

    for _ in range(3):
        fused()
        separate()
    ms_f = timed(fused, steps, torch.cuda.synchronize) / steps
    ms_s = timed(separate, steps, torch.cuda.synchronize) / steps
    fl = 14.0 * D * E
    return {"workload": f"{w.name} S{w.seq} with the L2Clip of q (learned scales, tau, threshold 9), fwd+bwd",
            "fused_ms": round(ms_f, 4), "separate_ms": round(ms_s, 4),
            "fused_tflops": round(fl / (ms_f * 1e-3) / 1e12, 1), "separate_tflops": round(fl / (ms_s * 1e-3) / 1e12, 1)}


def run_config(w, x, E, flops_step, world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": (f"{w.name}: B{w.batch} S{w.seq} Hq{w.heads_q} Hkv{w.heads_kv} D{w.head_dim} "
                         f"W{w.window} R{w.rel_extent} docs{w.docs} pad{w.pad}, {'fwd+bwd' if w.backward else 'fwd'}"),
            "global_batch": w.batch * world, "seq_len": w.seq, "parallelism": f"replicas x{world}",
            "allowed_elements": E, "flops_per_step": flops_step,
            "counts": ("allowed_elements and flops_per_step are one rank's batch; each rank draws its own "
                       "documents and value sums the FLOPs of all ranks" if world > 1 else "one GPU"),
            "l2": "inputs larger than L2 (profiles %.2f GB/step)" % (x["profiles"].numel() * 2 / 1e9)}


def run_reference(args, w, backward):
    """The oracle as the reference arm: each step is the FP64 oracle forward+backward
    on a bounded sample of the same workload, on the host cores."""
    from learned_relative_gqa_b200 import workloads
    x = workloads.make_inputs(w, "cpu")
    D = w.head_dim
    E_full = workloads.allowed_counts(w, x)
    threads = oracle_threads()
    s_sub, hc, E, dt = calibrate_sample(x, target_s=4.0, max_s=15.0)
    for _ in range(min(args.warmup, 1)):
        oracle_sample_step(hc)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(hc)
    dt = (time.perf_counter() - t0) / args.steps
    value = 14.0 * D * E / dt / 1e12
    G = hc["q"].shape[2]
    sample = (f"FP64 oracle forward+backward on batch 0, one KV group ({G} query heads), first {s_sub} tokens of "
              f"the same workload (E={E} allowed elements)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(w, x, E_full, (14.0 if backward else 4.0) * D * E_full, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
