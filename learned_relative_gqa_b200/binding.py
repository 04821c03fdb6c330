"""Thin Python binding of ``libinkling_rel_attn.so``.

Argument marshalling only: every step of the attention runs in the library's
CUDA kernels. The functions carry the C entry points' names; tensors are
PyTorch device tensors (PyTorch supplies device memory and streams), passed
to the library as raw pointers. There is no fallback: if the library is
missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libinkling_rel_attn.so")

INKLING_OK = 0
INKLING_ERR_INVALID_ARG = 1
INKLING_ERR_UNSUPPORTED = 2
INKLING_ERR_MALFORMED_POSITIONS = 3
INKLING_ERR_TIMEOUT = 4
INKLING_ERR_CUDA = 5


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "batch", "seq_q", "seq_k", "heads_q", "heads_kv", "head_dim", "rel_extent", "window", "query_offset")]


class FlexDims(ctypes.Structure):
    """inkling_flex_attn_dims (include/inkling_flex_attn.h)."""
    _fields_ = [(n, ctypes.c_int64) for n in (
        "batch", "seq", "heads_q", "heads_kv", "head_dim", "mask_type", "fixed_block_size", "sliding_window",
        "eos_id", "enable_gqa")] + [("scale", ctypes.c_double)]


FLEX_MASK_TYPES = {"causal": 0, "block_causal": 1}


class L2ClipDims(ctypes.Structure):
    """inkling_l2clip_dims (include/inkling_l2clip.h)."""
    _fields_ = [(n, ctypes.c_int64) for n in ("batch", "seq", "heads", "head_dim")] + [("threshold", ctypes.c_double)]


class InklingError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)} (status {status})"
        if status == INKLING_ERR_CUDA:
            msg += f": {load().inkling_rel_attn_last_cuda_error().decode()}"
        super().__init__(msg)


_lib = None


def load(path: str = LIB_PATH):
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{os.path.basename(path)} is not built; run python -m learned_relative_gqa_b200.build")
    lib = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    dp = ctypes.POINTER(Dims)
    lib.inkling_rel_attn_workspace_size.restype = sz
    lib.inkling_rel_attn_workspace_size.argtypes = [dp, ctypes.c_int]
    lib.inkling_rel_attn_validate.restype = ctypes.c_int
    lib.inkling_rel_attn_validate.argtypes = [dp, vp, vp, vp, vp, vp, sz, vp]
    lib.inkling_rel_attn_fwd.restype = ctypes.c_int
    lib.inkling_rel_attn_fwd.argtypes = [dp] + [vp] * 11 + [vp, sz, vp]
    lib.inkling_rel_attn_bwd.restype = ctypes.c_int
    lib.inkling_rel_attn_bwd.argtypes = [dp] + [vp] * 18 + [vp, sz, vp]
    lib.inkling_rel_attn_fwd_noalloc.restype = ctypes.c_int
    lib.inkling_rel_attn_fwd_noalloc.argtypes = [dp] + [vp] * 11 + [vp]
    lib.inkling_rel_attn_fwd_noalloc_last_device_error.restype = ctypes.c_int
    lib.inkling_rel_attn_fwd_noalloc_last_device_error.argtypes = [vp]
    lib.inkling_rel_attn_merge.restype = ctypes.c_int
    lib.inkling_rel_attn_merge.argtypes = [ctypes.c_int64, ctypes.c_int64, vp, vp, vp, vp, vp]
    lib.inkling_rel_attn_last_device_error.restype = ctypes.c_int
    lib.inkling_rel_attn_last_device_error.argtypes = [vp, vp]
    lib.inkling_rel_attn_selftest_exp2.restype = ctypes.c_int
    lib.inkling_rel_attn_selftest_exp2.argtypes = [vp, vp, ctypes.c_int64, vp]
    lib.inkling_rel_attn_selftest_wait_timeout.restype = ctypes.c_int
    lib.inkling_rel_attn_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp, sz, vp]
    lib.inkling_rel_attn_set_wait_timeout_ns.restype = ctypes.c_int
    lib.inkling_rel_attn_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.inkling_rel_attn_set_timing_events.restype = ctypes.c_int
    lib.inkling_rel_attn_set_timing_events.argtypes = [vp, ctypes.c_int]
    fd = ctypes.POINTER(FlexDims)
    lib.inkling_flex_attn_workspace_size.restype = sz
    lib.inkling_flex_attn_workspace_size.argtypes = [fd, ctypes.c_int]
    lib.inkling_flex_attn_fwd.restype = ctypes.c_int
    lib.inkling_flex_attn_fwd.argtypes = [fd] + [vp] * 7 + [vp, sz, vp]
    lib.inkling_flex_attn_bwd.restype = ctypes.c_int
    lib.inkling_flex_attn_bwd.argtypes = [fd] + [vp] * 12 + [vp, sz, vp]
    ld = ctypes.POINTER(L2ClipDims)
    lib.inkling_l2clip_workspace_size.restype = sz
    lib.inkling_l2clip_workspace_size.argtypes = [ld]
    lib.inkling_l2clip_fwd.restype = ctypes.c_int
    lib.inkling_l2clip_fwd.argtypes = [ld] + [vp] * 4 + [vp]
    lib.inkling_l2clip_bwd.restype = ctypes.c_int
    lib.inkling_l2clip_bwd.argtypes = [ld] + [vp] * 7 + [vp, sz, vp]
    lib.inkling_rel_attn_qclip_workspace_size.restype = sz
    lib.inkling_rel_attn_qclip_workspace_size.argtypes = [dp, ctypes.c_int]
    lib.inkling_rel_attn_fwd_qclip.restype = ctypes.c_int
    lib.inkling_rel_attn_fwd_qclip.argtypes = [dp, ctypes.c_double] + [vp] * 14 + [vp, sz, vp]
    lib.inkling_rel_attn_bwd_qclip.restype = ctypes.c_int
    lib.inkling_rel_attn_bwd_qclip.argtypes = [dp, ctypes.c_double] + [vp] * 23 + [vp, sz, vp]
    lib.inkling_rel_attn_last_cuda_error.restype = ctypes.c_char_p
    lib.inkling_rel_attn_last_cuda_error.argtypes = []
    lib.inkling_status_string.restype = ctypes.c_char_p
    lib.inkling_status_string.argtypes = [ctypes.c_int]
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().inkling_status_string(int(status)).decode()


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_dims(q: torch.Tensor, k: torch.Tensor, profiles: Optional[torch.Tensor], window: int,
              query_offset: int = 0, rel_extent: Optional[int] = None) -> Dims:
    B, S, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    R = profiles.shape[3] if profiles is not None else int(rel_extent or 0)
    return Dims(B, S, Skv, Hq, Hkv, D, R, int(window), int(query_offset))


def inkling_rel_attn_workspace_size(dims: Dims, backward: bool) -> int:
    return int(load().inkling_rel_attn_workspace_size(ctypes.byref(dims), int(bool(backward))))


def alloc_workspace(dims: Dims, backward: bool, device) -> torch.Tensor:
    n = inkling_rel_attn_workspace_size(dims, backward)
    if n == 0:
        raise InklingError(INKLING_ERR_INVALID_ARG, "workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _u8(t):
    return None if t is None else (t if t.dtype == torch.uint8 else t.view(torch.uint8) if t.dtype == torch.bool
                                   else t.to(torch.uint8))


def _check(status: int, where: str):
    if status != INKLING_OK:
        raise InklingError(status, where)


def inkling_rel_attn_validate(dims: Dims, valid, key_valid, positions, key_positions, workspace,
                              stream=None) -> int:
    """Returns the library status (INKLING_OK or INKLING_ERR_MALFORMED_POSITIONS, ...)."""
    return int(load().inkling_rel_attn_validate(
        ctypes.byref(dims), _p(_u8(valid)), _p(_u8(key_valid)), _p(positions), _p(key_positions),
        _p(workspace), workspace.numel(), _stream(stream)))


def inkling_rel_attn_fwd(dims: Dims, q, k, v, profiles, sink, valid, key_valid, positions, key_positions,
                         out, lse, workspace, stream=None) -> None:
    st = load().inkling_rel_attn_fwd(
        ctypes.byref(dims), _p(q), _p(k), _p(v), _p(profiles), _p(sink), _p(_u8(valid)), _p(_u8(key_valid)),
        _p(positions), _p(key_positions), _p(out), _p(lse), _p(workspace), workspace.numel(), _stream(stream))
    _check(st, "inkling_rel_attn_fwd")


def inkling_rel_attn_bwd(dims: Dims, q, k, v, profiles, sink, valid, key_valid, positions, key_positions,
                         out, lse, dout, dlse, dq, dk, dv, dprofiles, dsink, workspace, stream=None) -> None:
    st = load().inkling_rel_attn_bwd(
        ctypes.byref(dims), _p(q), _p(k), _p(v), _p(profiles), _p(sink), _p(_u8(valid)), _p(_u8(key_valid)),
        _p(positions), _p(key_positions), _p(out), _p(lse), _p(dout), _p(dlse), _p(dq), _p(dk), _p(dv),
        _p(dprofiles), _p(dsink), _p(workspace), workspace.numel(), _stream(stream))
    _check(st, "inkling_rel_attn_bwd")


def inkling_rel_attn_fwd_noalloc(dims: Dims, q, k, v, profiles, sink, valid, key_valid, positions, key_positions,
                                 out, lse, stream=None) -> int:
    """Forward that uses the library's own static device scratch instead of a workspace.

    For callers that cannot allocate device memory. Returns the library status
    (INKLING_ERR_UNSUPPORTED when the problem needs more than the 4 MiB of scratch).
    """
    return int(load().inkling_rel_attn_fwd_noalloc(
        ctypes.byref(dims), _p(q), _p(k), _p(v), _p(profiles), _p(sink), _p(_u8(valid)), _p(_u8(key_valid)),
        _p(positions), _p(key_positions), _p(out), _p(lse), _stream(stream)))


def inkling_rel_attn_merge(out, lse, out_part, lse_part, stream=None) -> None:
    """Merges (out_part, lse_part), a result over a disjoint key set, into (out, lse) in place."""
    for t in (out, lse, out_part, lse_part):
        if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()):
            raise ValueError("inkling_rel_attn_merge: contiguous float32 CUDA tensors expected")
    if out.shape != out_part.shape or lse.shape != lse_part.shape or out.shape[:-1] != lse.shape:
        raise ValueError("inkling_rel_attn_merge: shape mismatch")
    _check(load().inkling_rel_attn_merge(int(lse.numel()), int(out.shape[-1]), _p(out), _p(lse), _p(out_part),
                                         _p(lse_part), _stream(stream)), "inkling_rel_attn_merge")


def inkling_rel_attn_fwd_noalloc_last_device_error(stream=None) -> int:
    """Reads and clears the device error word of the no-allocation forward (synchronous)."""
    return int(load().inkling_rel_attn_fwd_noalloc_last_device_error(_stream(stream)))


def inkling_rel_attn_last_device_error(workspace, stream=None) -> int:
    return int(load().inkling_rel_attn_last_device_error(_p(workspace), _stream(stream)))


def inkling_rel_attn_selftest_wait_timeout(timeout_us: int, workspace, stream=None) -> int:
    return int(load().inkling_rel_attn_selftest_wait_timeout(int(timeout_us), _p(workspace), workspace.numel(),
                                                             _stream(stream)))


def inkling_rel_attn_set_wait_timeout_ns(timeout_ns: int) -> None:
    """Limit of the attention kernels' pipeline waits for later calls (0 = default)."""
    _check(load().inkling_rel_attn_set_wait_timeout_ns(int(timeout_ns)), "inkling_rel_attn_set_wait_timeout_ns")


def inkling_rel_attn_selftest_exp2(t, out, stream=None) -> None:
    """t, out: contiguous float32 CUDA tensors of the same size."""
    _check(load().inkling_rel_attn_selftest_exp2(_p(t), _p(out), int(t.numel()), _stream(stream)),
           "inkling_rel_attn_selftest_exp2")


def inkling_rel_attn_set_timing_events(events, n_pairs: int) -> None:
    """events: a ctypes array of cudaEvent_t handles (or None to switch the hook off)."""
    _check(load().inkling_rel_attn_set_timing_events(events, int(n_pairs)), "inkling_rel_attn_set_timing_events")


# --------------------------------------------------------------------------
# convenience wrappers (allocate outputs with torch, then call the entry points)
# --------------------------------------------------------------------------
def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")


def forward(q, k, v, profiles, sink, valid, key_valid=None, positions=None, key_positions=None, *,
            window: int = 0, query_offset: int = 0, workspace=None, stream=None):
    """out [B,S,Hq,D] fp32 and lse [B,S,Hq] fp32 (see include/inkling_rel_attn.h)."""
    _contig(q, k, v, profiles, sink, valid, key_valid, positions, key_positions)
    dims = make_dims(q, k, profiles, window, query_offset)
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    ws = alloc_workspace(dims, False, q.device) if workspace is None else workspace
    inkling_rel_attn_fwd(dims, q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, ws,
                         stream)
    return out, lse


def backward(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout, dlse=None, *,
             window: int = 0, query_offset: int = 0, workspace=None, stream=None):
    """dict dq, dk, dv, dprofiles, dsink (fp32)."""
    _contig(q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout, dlse)
    dims = make_dims(q, k, profiles, window, query_offset)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty(q.shape, **f32)
    dk = torch.empty(k.shape, **f32)
    dv = torch.empty(v.shape, **f32)
    dprof = torch.empty(profiles.shape, **f32)
    dsink = torch.empty(sink.shape, **f32)
    ws = alloc_workspace(dims, True, q.device) if workspace is None else workspace
    inkling_rel_attn_bwd(dims, q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout,
                         dlse, dq, dk, dv, dprof, dsink, ws, stream)
    return dict(dq=dq, dk=dk, dv=dv, dprofiles=dprof, dsink=dsink)


# --------------------------------------------------------------------------
# L2Clip of q fused into the attention (include/inkling_l2clip.h, *_qclip)
# --------------------------------------------------------------------------
def forward_qclip(x, k, v, profiles, sink, valid, key_valid=None, positions=None, key_positions=None, *,
                  threshold: float, clip_scale=None, tau=None, window: int = 0, query_offset: int = 0,
                  workspace=None, stream=None):
    """out [B,S,Hq,D] fp32, lse [B,S,Hq] fp32 and the clipped q [B,S,Hq,D] BF16 of the
    attention with q = L2Clip(x) computed inside the kernels."""
    _contig(x, k, v, profiles, sink, valid, key_valid, positions, key_positions, clip_scale, tau)
    dims = make_dims(x, k, profiles, window, query_offset)
    out = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    lse = torch.empty(x.shape[:3], dtype=torch.float32, device=x.device)
    qc = torch.empty_like(x)
    if workspace is None:
        workspace = torch.empty(max(int(load().inkling_rel_attn_qclip_workspace_size(ctypes.byref(dims), 0)), 256),
                                dtype=torch.uint8, device=x.device)
    st = load().inkling_rel_attn_fwd_qclip(
        ctypes.byref(dims), float(threshold), _p(clip_scale), _p(tau), _p(x), _p(k), _p(v), _p(profiles), _p(sink),
        _p(_u8(valid)), _p(_u8(key_valid)), _p(positions), _p(key_positions), _p(qc), _p(out), _p(lse),
        _p(workspace), workspace.numel(), _stream(stream))
    _check(st, "inkling_rel_attn_fwd_qclip")
    return out, lse, qc


def backward_qclip(x, q_clipped, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout,
                   dlse=None, *, threshold: float, clip_scale=None, tau=None, window: int = 0, query_offset: int = 0,
                   workspace=None, stream=None):
    """dict dx (gradient of the unclipped q), dk, dv, dprofiles, dsink, dclip_scale, dtau (fp32;
    the last two None without their parameters)."""
    _contig(x, q_clipped, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout, dlse,
            clip_scale, tau)
    dims = make_dims(x, k, profiles, window, query_offset)
    f32 = dict(dtype=torch.float32, device=x.device)
    g = dict(dx=torch.empty(x.shape, **f32), dk=torch.empty(k.shape, **f32), dv=torch.empty(v.shape, **f32),
             dprofiles=torch.empty(profiles.shape, **f32), dsink=torch.empty(sink.shape, **f32),
             dclip_scale=None if clip_scale is None else torch.empty(clip_scale.shape, **f32),
             dtau=None if tau is None else torch.empty(tau.shape, **f32))
    if workspace is None:
        workspace = torch.empty(int(load().inkling_rel_attn_qclip_workspace_size(ctypes.byref(dims), 1)),
                                dtype=torch.uint8, device=x.device)
    st = load().inkling_rel_attn_bwd_qclip(
        ctypes.byref(dims), float(threshold), _p(clip_scale), _p(tau), _p(x), _p(q_clipped), _p(k), _p(v),
        _p(profiles), _p(sink), _p(_u8(valid)), _p(_u8(key_valid)), _p(positions), _p(key_positions), _p(out),
        _p(lse), _p(dout), _p(dlse), _p(g["dx"]), _p(g["dk"]), _p(g["dv"]), _p(g["dprofiles"]), _p(g["dsink"]),
        _p(g["dclip_scale"]), _p(g["dtau"]), _p(workspace), workspace.numel(), _stream(stream))
    _check(st, "inkling_rel_attn_bwd_qclip")
    return g


# --------------------------------------------------------------------------
# generic FlexAttention variant (include/inkling_flex_attn.h)
# --------------------------------------------------------------------------
def make_flex_dims(q: torch.Tensor, k: torch.Tensor, *, mask_type: str = "causal", eos_id: int = 0,
                   fixed_block_size: int = 0, sliding_window: int = 0, scale: Optional[float] = None,
                   enable_gqa: bool = False) -> FlexDims:
    B, Hq, S, D = q.shape
    if mask_type not in FLEX_MASK_TYPES:
        raise ValueError(f"mask_type must be one of {sorted(FLEX_MASK_TYPES)}")
    return FlexDims(B, S, Hq, k.shape[1], D, FLEX_MASK_TYPES[mask_type], int(fixed_block_size), int(sliding_window),
                    int(eos_id), int(bool(enable_gqa)), 0.0 if scale is None else float(scale))


def inkling_flex_attn_workspace_size(dims: FlexDims, backward: bool) -> int:
    return int(load().inkling_flex_attn_workspace_size(ctypes.byref(dims), int(bool(backward))))


def inkling_flex_attn_fwd(dims: FlexDims, q, k, v, sink_weights, tokens, out, lse, workspace, stream=None) -> None:
    st = load().inkling_flex_attn_fwd(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(sink_weights), _p(tokens), _p(out),
                                      _p(lse), _p(workspace), workspace.numel(), _stream(stream))
    _check(st, "inkling_flex_attn_fwd")


def inkling_flex_attn_bwd(dims: FlexDims, q, k, v, sink_weights, tokens, out, lse, dout, dq, dk, dv, dsink_weights,
                          workspace, stream=None) -> None:
    st = load().inkling_flex_attn_bwd(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(sink_weights), _p(tokens),
                                      _p(out), _p(lse), _p(dout), _p(dq), _p(dk), _p(dv), _p(dsink_weights),
                                      _p(workspace), workspace.numel(), _stream(stream))
    _check(st, "inkling_flex_attn_bwd")


def _flex_ws(dims: FlexDims, backward: bool, device) -> torch.Tensor:
    n = inkling_flex_attn_workspace_size(dims, backward)
    if n == 0:
        raise InklingError(INKLING_ERR_INVALID_ARG, "inkling_flex_attn_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def flex_forward(q, k, v, sink_weights=None, tokens=None, *, mask_type: str = "causal", eos_id: int = 0,
                 fixed_block_size: int = 0, sliding_window: int = 0, scale: Optional[float] = None,
                 enable_gqa: bool = False, workspace=None, stream=None):
    """out [B,Hq,S,D] BF16 and lse [B,Hq,S] FP32 (see include/inkling_flex_attn.h)."""
    _contig(q, k, v, sink_weights, tokens)
    dims = make_flex_dims(q, k, mask_type=mask_type, eos_id=eos_id, fixed_block_size=fixed_block_size,
                          sliding_window=sliding_window, scale=scale, enable_gqa=enable_gqa)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    ws = _flex_ws(dims, False, q.device) if workspace is None else workspace
    inkling_flex_attn_fwd(dims, q, k, v, sink_weights, tokens, out, lse, ws, stream)
    return out, lse


def flex_backward(q, k, v, out, lse, dout, sink_weights=None, tokens=None, *, mask_type: str = "causal",
                  eos_id: int = 0, fixed_block_size: int = 0, sliding_window: int = 0,
                  scale: Optional[float] = None, enable_gqa: bool = False, workspace=None, stream=None):
    """dict dq [B,Hq,S,D], dk / dv [B,Hkv,S,D] and dsink_weights [Hq] (None without sinks), FP32."""
    _contig(q, k, v, out, lse, dout, sink_weights, tokens)
    dims = make_flex_dims(q, k, mask_type=mask_type, eos_id=eos_id, fixed_block_size=fixed_block_size,
                          sliding_window=sliding_window, scale=scale, enable_gqa=enable_gqa)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty(q.shape, **f32)
    dk = torch.empty(k.shape, **f32)
    dv = torch.empty(v.shape, **f32)
    dsw = None if sink_weights is None else torch.empty(sink_weights.shape, **f32)
    ws = _flex_ws(dims, True, q.device) if workspace is None else workspace
    inkling_flex_attn_bwd(dims, q, k, v, sink_weights, tokens, out, lse, dout, dq, dk, dv, dsw, ws, stream)
    return dict(dq=dq, dk=dk, dv=dv, dsink_weights=dsw)


# --------------------------------------------------------------------------
# L2Clip (include/inkling_l2clip.h)
# --------------------------------------------------------------------------
def make_l2clip_dims(x: torch.Tensor, threshold: float) -> L2ClipDims:
    B, S, H, D = x.shape
    return L2ClipDims(B, S, H, D, float(threshold))


def inkling_l2clip_workspace_size(dims: L2ClipDims) -> int:
    return int(load().inkling_l2clip_workspace_size(ctypes.byref(dims)))


def inkling_l2clip_fwd(dims: L2ClipDims, x, scale, tau, y, stream=None) -> None:
    _check(load().inkling_l2clip_fwd(ctypes.byref(dims), _p(x), _p(scale), _p(tau), _p(y), _stream(stream)),
           "inkling_l2clip_fwd")


def inkling_l2clip_bwd(dims: L2ClipDims, x, scale, tau, dy, dx, dscale, dtau, workspace, stream=None) -> None:
    _check(load().inkling_l2clip_bwd(ctypes.byref(dims), _p(x), _p(scale), _p(tau), _p(dy), _p(dx), _p(dscale),
                                     _p(dtau), _p(workspace), workspace.numel(), _stream(stream)),
           "inkling_l2clip_bwd")


def l2clip_forward(x, threshold: float, scale=None, tau=None, stream=None):
    """y [B,S,H,D] BF16: x (BF16) clipped per head vector (see include/inkling_l2clip.h)."""
    _contig(x, scale, tau)
    dims = make_l2clip_dims(x, threshold)
    y = torch.empty_like(x)
    inkling_l2clip_fwd(dims, x, scale, tau, y, stream)
    return y


def l2clip_backward(x, dy, threshold: float, scale=None, tau=None, stream=None):
    """dict dx [B,S,H,D], dscale [H,D] (None without scale), dtau [B,S] (None without tau), FP32."""
    _contig(x, dy, scale, tau)
    dims = make_l2clip_dims(x, threshold)
    f32 = dict(dtype=torch.float32, device=x.device)
    dx = torch.empty(x.shape, **f32)
    dscale = None if scale is None else torch.empty(scale.shape, **f32)
    dtau = None if tau is None else torch.empty(tau.shape, **f32)
    n = inkling_l2clip_workspace_size(dims)
    if n == 0:
        raise InklingError(INKLING_ERR_INVALID_ARG, "inkling_l2clip_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=x.device)
    inkling_l2clip_bwd(dims, x, scale, tau, dy, dx, dscale, dtau, ws, stream)
    return dict(dx=dx, dscale=dscale, dtau=dtau)

