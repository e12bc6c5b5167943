"""LLM.int8() forward linear layer for B200 (sm_100a).

The compute lives in the C-ABI library ``libint8mp.so`` built from
``csrc/``; ``int8_mixed_precision_column_b200.native`` is the thin ctypes
binding over it.  The binding is imported lazily so that the seeded input
generators in ``workloads`` stay importable on machines without a GPU.
"""

__all__ = ["native", "workloads"]


def __getattr__(name):
    if name == "native":
        from . import native

        return native
    raise AttributeError(name)
