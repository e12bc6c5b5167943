"""LLM.int8() forward linear layer for B200 (sm_100a).

The compute lives in the C-ABI library ``libint8mp.so`` built from
``csrc/`` by ``build.py``; ``native`` is the thin ctypes binding over it
(the library is loaded on first use, so importing the package needs no GPU).
``workloads`` holds the seeded synthetic input generators.
"""

__all__ = ["build", "native", "workloads"]
