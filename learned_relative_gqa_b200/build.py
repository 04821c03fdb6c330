"""Build libinkling_rel_attn.so in-tree with nvcc for sm_100a.

Usage: ``python -m learned_relative_gqa_b200.build [--verbose]``.
The library is written next to this file; nothing is installed elsewhere.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libinkling_rel_attn.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
# the same kernels with every shared / global index checked (-DINKLING_BOUNDS_CHECK), for tests
BOUNDS_CHECK_LIB_PATH = os.path.join(HERE, "libinkling_rel_attn_boundscheck.so")
SOURCES = ["host.cu", "prep_kernels.cu", "fwd.cu", "bwd.cu", "l2clip.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale(path: str = LIB_PATH) -> bool:
    """True when the library at `path` is missing or older than a source or header."""
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return any(os.path.getmtime(d) > t for d in deps)


_stale = stale


def build(force: bool = False, verbose: bool = False, out_path: str = LIB_PATH, defines: tuple = ()) -> str:
    """Compile the library. ``defines`` / ``out_path`` build diagnostic variants
    (for example ``INKLING_TRACE``) next to, not over, the product library."""
    if not force and not defines and out_path == LIB_PATH and not _stale():
        return LIB_PATH
    objs = []
    build_dir = os.path.join(ROOT, "_build", "-".join(defines) or "default")
    os.makedirs(build_dir, exist_ok=True)
    common = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INCLUDE,
              "--expt-relaxed-constexpr"]
    if verbose:
        common += ["-Xptxas", "-v"]
    common += [f"-D{d}" for d in defines]
    procs = []
    for src in SOURCES:  # translation units compile side by side
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        procs.append((subprocess.Popen(common + ["-c", os.path.join(CSRC, src), "-o", obj]), src))
        objs.append(obj)
    failed = [src for proc, src in procs if proc.wait() != 0]
    if failed:
        raise RuntimeError(f"nvcc failed on {', '.join(failed)}")
    tmp = out_path + ".tmp"
    subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs], check=True)
    os.replace(tmp, out_path)
    return out_path


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
