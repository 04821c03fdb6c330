"""FP64 CPU oracle for Inkling2 learned-relative GQA attention.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers. The product path never imports this
package, and this package imports nothing from the product path; the two
share only the seeded input generator (which holds none of the method's
arithmetic), and even that is passed in as plain arrays here.

The arithmetic lives in ``rel_attn_oracle.c`` (plain C, double precision,
OpenMP over independent rows); this module compiles it with gcc, loads it
with ctypes and marshals numpy arrays. Semantics follow the NeMo AutoModel
API pages for ``Inkling2FlexAttention.forward`` (argument list, shapes,
defaults) and ``Inkling2Attention._eager`` (the quadratic reference).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rel_attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "batch", "seq_q", "seq_k", "heads_q", "heads_kv", "head_dim", "rel_extent",
        "window", "query_offset", "window_inclusive")]


def build(out_path: str = _LIB_PATH, defines: tuple = (), force: bool = False) -> str:
    """Compile the oracle C source into a shared library (gcc, -O2, OpenMP).

    ``defines`` adds ``-D`` flags; the mutation self-tests use it to build
    deliberately broken variants under a different ``out_path``.
    """
    if (not force and not defines and os.path.exists(out_path)
            and os.path.getmtime(out_path) >= os.path.getmtime(_SRC)):
        return out_path
    cmd = ["gcc", "-O2", "-fopenmp", "-std=c11", "-shared", "-fPIC", "-o", out_path, _SRC, "-lm"]
    cmd[1:1] = [f"-D{d}" for d in defines]
    subprocess.run(cmd, check=True)
    return out_path


def _bind(lib):
    vp = ctypes.c_void_p
    lib.oracle_fwd_f64.restype = ctypes.c_int
    lib.oracle_fwd_f64.argtypes = [ctypes.POINTER(_Dims)] + [vp] * 12 + [vp, ctypes.c_int64]
    lib.oracle_bwd_f64.restype = ctypes.c_int
    lib.oracle_bwd_f64.argtypes = [ctypes.POINTER(_Dims)] + [vp] * 16
    lib.oracle_bwd_sampled_f64.restype = ctypes.c_int
    lib.oracle_bwd_sampled_f64.argtypes = ([ctypes.POINTER(_Dims)] + [vp] * 11
                                           + [vp, ctypes.c_int64, vp, ctypes.c_int64] + [vp] * 5)
    lib.oracle_set_threads.restype = None
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_threads.restype = ctypes.c_int
    lib.oracle_threads.argtypes = []
    lib.oracle_decode_bf16.restype = None
    lib.oracle_decode_bf16.argtypes = [vp, vp, ctypes.c_int64]
    return lib


def load(path: Optional[str] = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


# --------------------------------------------------------------------------
# marshalling helpers
# --------------------------------------------------------------------------
def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def set_threads(n: int) -> int:
    """Use n OpenMP threads in the oracle's parallel loops; returns the count now in effect."""
    lib = load()
    lib.oracle_set_threads(int(n))
    return int(lib.oracle_threads())


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """Exact BF16 bit patterns (uint16/int16) -> float64, decoded by the oracle's own C routine."""
    src = np.ascontiguousarray(np.asarray(bits).view(np.uint16))
    dst = np.empty(src.shape, dtype=np.float64)
    load().oracle_decode_bf16(_ptr(src), _ptr(dst), src.size)
    return dst


def resolve_defaults(valid, key_valid, positions, key_positions, seq_k: int, query_offset: int):
    """Apply the forward() defaults of the API page.

    * ``key_valid`` None  -> ``valid`` (single-shard case: needs Skv == S and offset 0).
    * ``positions`` None -> one document: query_offset + arange(S).
    * ``key_positions`` None -> ``positions`` when they were given (needs Skv == S and
      offset 0), else arange(Skv).
    """
    valid = np.ascontiguousarray(np.asarray(valid, dtype=np.uint8))
    B, S = valid.shape
    if key_valid is None:
        if seq_k != S or query_offset != 0:
            raise ValueError("key_valid may default to valid only when Skv == S and query_offset == 0")
        key_valid = valid
    key_valid = np.ascontiguousarray(np.asarray(key_valid, dtype=np.uint8))
    pos_given = positions is not None
    if positions is None:
        positions = np.broadcast_to(np.arange(S, dtype=np.int32) + query_offset, (B, S))
    positions = np.ascontiguousarray(np.asarray(positions, dtype=np.int32))
    if key_positions is None:
        if pos_given:
            if seq_k != S or query_offset != 0:
                raise ValueError("key_positions may default to positions only when Skv == S and offset 0")
            key_positions = positions
        else:
            key_positions = np.broadcast_to(np.arange(seq_k, dtype=np.int32), (B, seq_k))
    key_positions = np.ascontiguousarray(np.asarray(key_positions, dtype=np.int32))
    return valid, key_valid, positions, key_positions


def _dims(q, k, profiles, window, query_offset, window_inclusive):
    B, S, Hq, D = q.shape
    _, Skv, Hkv, _ = k.shape
    R = profiles.shape[3]
    return _Dims(B, S, Skv, Hq, Hkv, D, R, int(window), int(query_offset), int(bool(window_inclusive)))


def forward(q, k, v, profiles, sink, valid, key_valid=None, positions=None, key_positions=None,
            *, window: int = 0, query_offset: int = 0, window_inclusive: bool = False,
            rows: Optional[np.ndarray] = None):
    """Quadratic FP64 forward.

    q [B,S,Hq,D], k/v [B,Skv,Hkv,D], profiles [B,Hq,S,R]: float64 values (decode BF16
    first with :func:`decode_bf16`); sink [B,S,Hq]; valid [B,S]; key_valid [B,Skv];
    positions [B,S]; key_positions [B,Skv].

    Returns (out [B,S,Hq,D], lse [B,S,Hq], lse_content [B,S,Hq]) in float64. When
    ``rows`` (flattened (b*S+i)*Hq+h ids) is given only those rows are computed and
    the other entries are NaN.
    """
    q, k, v, profiles, sink = map(_f64, (q, k, v, profiles, sink))
    dims = _dims(q, k, profiles, window, query_offset, window_inclusive)
    valid, key_valid, positions, key_positions = resolve_defaults(
        valid, key_valid, positions, key_positions, k.shape[1], query_offset)
    fill = np.nan if rows is not None else 0.0
    out = np.full(q.shape, fill)
    lse = np.full(q.shape[:3], fill)
    lsec = np.full(q.shape[:3], fill)
    rows_arr = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    rc = load().oracle_fwd_f64(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(profiles), _ptr(sink),
                               _ptr(valid), _ptr(key_valid), _ptr(positions), _ptr(key_positions),
                               _ptr(out), _ptr(lse), _ptr(lsec), _ptr(rows_arr),
                               0 if rows_arr is None else rows_arr.size)
    if rc:
        raise ValueError(f"oracle_fwd_f64 rejected the dimensions (code {rc})")
    return out, lse, lsec


def backward(q, k, v, profiles, sink, valid, key_valid=None, positions=None, key_positions=None,
             *, dout, dlse=None, window: int = 0, query_offset: int = 0, window_inclusive: bool = False):
    """Full FP64 backward. Returns dict dq, dk, dv, dprofiles, dsink (float64)."""
    q, k, v, profiles, sink, dout = map(_f64, (q, k, v, profiles, sink, dout))
    dlse = None if dlse is None else _f64(dlse)
    dims = _dims(q, k, profiles, window, query_offset, window_inclusive)
    valid, key_valid, positions, key_positions = resolve_defaults(
        valid, key_valid, positions, key_positions, k.shape[1], query_offset)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    dprof = np.zeros(profiles.shape)
    dsink = np.zeros(sink.shape)
    rc = load().oracle_bwd_f64(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(profiles), _ptr(sink),
                               _ptr(valid), _ptr(key_valid), _ptr(positions), _ptr(key_positions),
                               _ptr(dout), _ptr(dlse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dprof),
                               _ptr(dsink))
    if rc:
        raise ValueError(f"oracle_bwd_f64 rejected the dimensions (code {rc})")
    return dict(dq=dq, dk=dk, dv=dv, dprofiles=dprof, dsink=dsink)


def backward_sampled(q, k, v, profiles, sink, valid, key_valid=None, positions=None, key_positions=None,
                     *, dout, dlse=None, rows=(), keys=(), window: int = 0, query_offset: int = 0):
    """Sampled FP64 backward for large shapes.

    ``rows``: flattened query-row ids (b*S+i)*Hq+h -> dq, dprofiles, dsink rows.
    ``keys``: flattened key ids (b*Skv+j)*Hkv+g -> dk, dv rows.
    Entries outside the samples are NaN.
    """
    q, k, v, profiles, sink, dout = map(_f64, (q, k, v, profiles, sink, dout))
    dlse = None if dlse is None else _f64(dlse)
    dims = _dims(q, k, profiles, window, query_offset, False)
    valid, key_valid, positions, key_positions = resolve_defaults(
        valid, key_valid, positions, key_positions, k.shape[1], query_offset)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    dprof = np.full(profiles.shape, np.nan)
    dsink = np.full(sink.shape, np.nan)
    rc = load().oracle_bwd_sampled_f64(
        ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(profiles), _ptr(sink),
        _ptr(valid), _ptr(key_valid), _ptr(positions), _ptr(key_positions), _ptr(dout), _ptr(dlse),
        _ptr(rows), rows.size, _ptr(keys), keys.size,
        _ptr(dq), _ptr(dprof), _ptr(dsink), _ptr(dk), _ptr(dv))
    if rc:
        raise ValueError(f"oracle_bwd_sampled_f64 rejected the dimensions (code {rc})")
    return dict(dq=dq, dk=dk, dv=dv, dprofiles=dprof, dsink=dsink)
