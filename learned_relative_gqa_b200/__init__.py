"""B200-native Inkling2 learned-relative grouped-query attention.

The hot path (forward and backward) is hand-written CUDA for sm_100a behind a
C-ABI shared library (``libinkling_rel_attn.so``, declared in
``include/inkling_rel_attn.h``). This package holds that library's sources
(``csrc/``), a thin ctypes binding with the same entry-point names
(:mod:`learned_relative_gqa_b200.binding`) and the seeded synthetic workloads
(:mod:`learned_relative_gqa_b200.workloads`). The binding is imported lazily
so that the workloads can be used on machines without the built library.
"""

__all__ = ["binding", "workloads"]


def __getattr__(name):
    if name in ("binding", "workloads"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
