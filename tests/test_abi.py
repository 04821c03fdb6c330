"""CPU-only checks of the C-ABI library: it builds, loads, exports every entry
point declared in include/*.h, sizes workspaces, and rejects bad arguments on
the host before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", n) for n in sorted(os.listdir(os.path.join(ROOT, "include")))
           if n.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    from learned_relative_gqa_b200 import build, binding
    build.build()
    return binding.load()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(inkling_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("inkling_rel_attn_fwd", "inkling_rel_attn_bwd", "inkling_rel_attn_validate",
                 "inkling_rel_attn_workspace_size", "inkling_rel_attn_last_device_error", "inkling_status_string",
                 "inkling_flex_attn_fwd", "inkling_flex_attn_bwd", "inkling_flex_attn_workspace_size"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_library_does_not_link_the_oracle(lib):
    from learned_relative_gqa_b200 import binding
    data = open(binding.LIB_PATH, "rb").read()
    assert b"oracle_fwd_f64" not in data and b"oracle_bwd_f64" not in data


def dims(**kw):
    from learned_relative_gqa_b200.binding import Dims
    base = dict(batch=2, seq_q=256, seq_k=256, heads_q=8, heads_kv=2, head_dim=128, rel_extent=64, window=0,
                query_offset=0)
    base.update(kw)
    return Dims(**base)


def test_workspace_size(lib):
    from learned_relative_gqa_b200.binding import inkling_rel_attn_workspace_size as ws
    f, b = ws(dims(), False), ws(dims(), True)
    assert 0 < f < b
    # backward holds a BF16 copy of dout plus two [B,Hq,S] fp32 arrays
    assert b - f >= 2 * 256 * 8 * 128 * 2 + 2 * 2 * 8 * 256 * 4
    assert ws(dims(seq_q=512, seq_k=512), False) > f
    assert ws(dims(head_dim=96), False) == 0
    assert ws(dims(heads_q=6, heads_kv=4), False) == 0
    assert ws(dims(rel_extent=12), False) == 0


@pytest.mark.parametrize("bad,expect", [
    (dict(head_dim=96), 2),
    (dict(rel_extent=12), 2),
    (dict(heads_q=6, heads_kv=4), 1),
    (dict(window=-1), 1),
    (dict(seq_q=-3), 1),
    # profile rows b * Hq * S + h * S + i must stay below 2^31 when R > 0
    (dict(batch=64, heads_q=64, heads_kv=8, seq_q=1 << 19, seq_k=1 << 19), 2),
])
def test_fwd_rejects_bad_dims_on_host(lib, bad, expect):
    d = dims(**bad)
    st = lib.inkling_rel_attn_fwd(ctypes.byref(d), *([None] * 11), None, 0, None)
    assert st == expect


def test_fwd_rejects_null_and_misaligned_pointers(lib):
    d = dims()
    fake = ctypes.c_void_p(0x10000)
    mis = ctypes.c_void_p(0x10008)
    args = [fake] * 11
    st = lib.inkling_rel_attn_fwd(ctypes.byref(d), None, *args[1:], fake, 1 << 30, None)
    assert st == 1  # null q
    st = lib.inkling_rel_attn_fwd(ctypes.byref(d), mis, *args[1:], fake, 1 << 30, None)
    assert st == 1  # misaligned q
    # workspace too small
    st = lib.inkling_rel_attn_fwd(ctypes.byref(d), *args, fake, 16, None)
    assert st == 1
    # key_valid may not default to valid under a query offset
    d2 = dims(query_offset=64, seq_k=320)
    a2 = list(args)
    a2[6] = None  # key_valid
    st = lib.inkling_rel_attn_fwd(ctypes.byref(d2), *a2, fake, 1 << 30, None)
    assert st == 1


def test_bwd_rejects_bad_arguments_on_host(lib):
    d = dims(head_dim=32)
    assert lib.inkling_rel_attn_bwd(ctypes.byref(d), *([None] * 18), None, 0, None) == 2
    d = dims()
    fake = ctypes.c_void_p(0x10000)
    args = [fake] * 18
    args[13] = None  # dlse is optional
    a = list(args)
    a[14] = None     # dq missing
    assert lib.inkling_rel_attn_bwd(ctypes.byref(d), *a, fake, 1 << 34, None) == 1


def test_status_strings(lib):
    from learned_relative_gqa_b200 import binding
    assert binding.status_string(0) == "ok"
    assert "timed out" in binding.status_string(4)
    assert binding.status_string(77) == "unknown status"


def flex_dims(**kw):
    from learned_relative_gqa_b200.binding import FlexDims
    base = dict(batch=2, seq=256, heads_q=8, heads_kv=2, head_dim=128, mask_type=1, fixed_block_size=0,
                sliding_window=0, eos_id=2, enable_gqa=1, scale=0.0)
    base.update(kw)
    return FlexDims(**base)


def test_flex_workspace_size(lib):
    from learned_relative_gqa_b200.binding import inkling_flex_attn_workspace_size as ws
    f, b = ws(flex_dims(), False), ws(flex_dims(), True)
    assert 0 < f < b
    assert ws(flex_dims(enable_gqa=0), False) == 0        # Hq != Hkv needs enable_gqa
    assert ws(flex_dims(heads_q=2, enable_gqa=0), False) > 0
    assert ws(flex_dims(mask_type=7), False) == 0
    assert ws(flex_dims(head_dim=80), False) == 0
    assert ws(flex_dims(sliding_window=-1), False) == 0


def test_flex_rejects_bad_arguments_on_host(lib):
    fake = ctypes.c_void_p(0x10000)
    d = flex_dims(head_dim=96)
    assert lib.inkling_flex_attn_fwd(ctypes.byref(d), *([fake] * 7), fake, 1 << 30, None) == 2
    d = flex_dims()
    a = [fake] * 7
    a[4] = None  # block_causal without tokens
    assert lib.inkling_flex_attn_fwd(ctypes.byref(d), *a, fake, 1 << 30, None) == 1
    a = [fake] * 7
    a[0] = ctypes.c_void_p(0x10008)  # misaligned q
    assert lib.inkling_flex_attn_fwd(ctypes.byref(d), *a, fake, 1 << 30, None) == 1
    assert lib.inkling_flex_attn_fwd(ctypes.byref(d), *([fake] * 7), fake, 64, None) == 1  # small workspace
    b = [fake] * 12
    b[11] = None  # sink weights without a place for their gradient
    assert lib.inkling_flex_attn_bwd(ctypes.byref(d), *b, fake, 1 << 34, None) == 1


def test_l2clip_rejects_bad_arguments_on_host(lib):
    from learned_relative_gqa_b200.binding import L2ClipDims
    fake = ctypes.c_void_p(0x10000)
    good = L2ClipDims(2, 64, 8, 128, 1.0)
    assert lib.inkling_l2clip_workspace_size(ctypes.byref(good)) > 0
    assert lib.inkling_l2clip_workspace_size(ctypes.byref(L2ClipDims(2, 64, 8, 96, 1.0))) == 0
    assert lib.inkling_l2clip_fwd(ctypes.byref(L2ClipDims(2, 64, 8, 128, -1.0)), fake, None, None, fake, None) == 1
    assert lib.inkling_l2clip_fwd(ctypes.byref(L2ClipDims(2, 64, 8, 128, float("nan"))), fake, None, None, fake,
                                  None) == 1
    assert lib.inkling_l2clip_fwd(ctypes.byref(good), None, None, None, fake, None) == 1
    assert lib.inkling_l2clip_fwd(ctypes.byref(good), ctypes.c_void_p(0x10004), None, None, fake, None) == 1
    # a learned scale needs a place for its gradient, and the reverse
    assert lib.inkling_l2clip_bwd(ctypes.byref(good), fake, fake, None, fake, fake, None, None, fake, 1 << 30,
                                  None) == 1
    assert lib.inkling_l2clip_bwd(ctypes.byref(good), fake, None, None, fake, fake, None, fake, fake, 1 << 30,
                                  None) == 1
    assert lib.inkling_l2clip_bwd(ctypes.byref(good), fake, None, None, fake, fake, None, None, fake, 16, None) == 1


def test_binding_fails_loudly_without_the_library(tmp_path):
    """No CPU or library fallback: a missing shared library raises on load."""
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from learned_relative_gqa_b200 import binding\n"
            "binding._lib = None\n"
            "try:\n"
            "    binding.load(%r)\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n"
            "else:\n"
            "    print('loaded')\n") % (ROOT, str(tmp_path / "libinkling_rel_attn.so"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.startswith("raised:") and "not built" in r.stdout


def test_product_modules_do_not_import_the_oracle():
    import ast
    pkg = os.path.join(ROOT, "learned_relative_gqa_b200")
    for name in os.listdir(pkg):
        if not name.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(pkg, name)).read())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                assert all(not a.name.startswith("oracle") for a in node.names), name
            elif isinstance(node, ast.ImportFrom):
                assert not (node.module or "").startswith("oracle"), name
