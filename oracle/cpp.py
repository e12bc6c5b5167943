"""The plain C++ oracle (``llm_int8_ref.cpp``) behind the numpy oracle's API.

TEST INFRASTRUCTURE ONLY: ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline of ``bench.py`` use it; the product path never does.  Every step of
the method runs in the C++ translation unit (plain loops, IEEE fp32 / fp64,
no intrinsics, no fast-math, no FMA contraction); this module only converts
numpy arrays to pointers and composes the steps in the order of the numpy
oracle (``oracle.llm_int8``), whose functions and returned dictionaries it
mirrors, so the same pins run on both.

``build()`` compiles the library with g++ into ``oracle/lib/``;
``Oracle(path)`` loads a build (a planted-mistake test loads a modified copy
compiled elsewhere).
"""

from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "llm_int8_ref.cpp")
LIB = os.path.join(HERE, "lib", "liboracle_ref.so")
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off", "-fno-fast-math"]
Q_MAX = 127
F16, BF16 = 0, 1


def compile_source(src: str, out: str) -> str:
    """g++ the oracle source ``src`` into the shared library ``out``."""
    cxx = os.environ.get("CXX") or shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        raise RuntimeError("no C++ compiler (g++) for the C++ oracle")
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + ".tmp"
    r = subprocess.run([cxx, *CXXFLAGS, src, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"building the C++ oracle failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``llm_int8_ref.cpp`` into ``oracle/lib/liboracle_ref.so`` when stale."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_source(SRC, LIB)


def _p(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


class Oracle:
    """The C++ oracle with the numpy oracle's functions (fp16 arrays as
    ``np.float16``, bf16 as uint16 bit patterns)."""

    Q_MAX = Q_MAX

    def __init__(self, path: str | None = None, threads: int | None = None):
        self.path = path or build()
        self.lib = ctypes.CDLL(self.path)
        self.threads = int(threads or os.cpu_count() or 1)
        L, P, I64, I = self.lib, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        sig = {
            "oref_to_f32": (None, [P, I64, I, P]),
            "oref_from_f32": (None, [P, I64, I, P]),
            "oref_quantize_weight": (None, [P, I64, I64, I, P, P, I]),
            "oref_outlier_mask": (None, [P, I64, I64, I, ctypes.c_float, P]),
            "oref_outlier_index": (I64, [P, I64, P]),
            "oref_quantize_rows": (None, [P, I64, I64, I, P, P, P, I]),
            "oref_outlier_operands": (None, [P, I64, I64, P, P, I64, P, I64, I, P, P]),
            "oref_int8_matmul": (None, [P, I64, I64, P, I64, P, I]),
            "oref_combine": (None, [P, P, P, P, P, I64, P, I, I64, I64, P, I]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args

    # -- 16-bit conversions --------------------------------------------------
    def to_f32(self, u16, elem: int) -> np.ndarray:
        a = np.ascontiguousarray(u16, dtype=np.uint16)
        out = np.empty(a.shape, np.float32)
        self.lib.oref_to_f32(_p(a), a.size, elem, _p(out))
        return out.reshape(np.shape(u16))

    def from_f32(self, x, elem: int) -> np.ndarray:
        a = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(a.shape, np.uint16)
        self.lib.oref_from_f32(_p(a), a.size, elem, _p(out))
        return out.reshape(np.shape(x))

    def bf16_to_f32(self, u16) -> np.ndarray:
        return self.to_f32(u16, BF16)

    def f32_to_bf16(self, x) -> np.ndarray:
        return self.from_f32(x, BF16)

    # -- the steps (16-bit operands as bit patterns, element type `elem`) ------
    def _quantize_weight(self, W16: np.ndarray, elem: int):
        W16 = np.ascontiguousarray(W16, dtype=np.uint16)
        N, K = W16.shape
        CB = np.empty((N, K), np.int8)
        SCB = np.empty(N, np.float32)
        self.lib.oref_quantize_weight(_p(W16), N, K, elem, _p(CB), _p(SCB), self.threads)
        return CB, SCB

    def _mask(self, X16: np.ndarray, threshold: float, elem: int) -> np.ndarray:
        X16 = np.ascontiguousarray(X16, dtype=np.uint16)
        T, K = X16.shape
        m = np.empty(K, np.uint8)
        self.lib.oref_outlier_mask(_p(X16), T, K, elem, float(threshold), _p(m))
        return m.astype(bool)

    def outlier_index(self, mask) -> np.ndarray:
        m = np.ascontiguousarray(mask, dtype=np.uint8)
        idx = np.empty(m.size, np.int32)
        n = self.lib.oref_outlier_index(_p(m), m.size, _p(idx))
        return idx[:n].copy()

    def _rows(self, X16: np.ndarray, mask, elem: int):
        X16 = np.ascontiguousarray(X16, dtype=np.uint16)
        T, K = X16.shape
        m = np.ascontiguousarray(mask, dtype=np.uint8)
        Xq = np.empty((T, K), np.int8)
        sA = np.empty(T, np.float32)
        self.lib.oref_quantize_rows(_p(X16), T, K, elem, _p(m), _p(Xq), _p(sA), self.threads)
        return Xq, sA

    def _operands(self, X16, CB, SCB, idx, elem: int):
        X16 = np.ascontiguousarray(X16, dtype=np.uint16)
        CB = np.ascontiguousarray(CB, dtype=np.int8)
        SCB = np.ascontiguousarray(SCB, dtype=np.float32)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        T, K = X16.shape
        N = CB.shape[0]
        n = idx.size
        Xo = np.empty((T, n), np.uint16)
        Wo = np.empty((N, n), np.uint16)
        self.lib.oref_outlier_operands(_p(X16), T, K, _p(CB), _p(SCB), N, _p(idx), n, elem, _p(Xo), _p(Wo))
        return Xo, Wo

    def int8_matmul(self, Xq, CB) -> np.ndarray:
        Xq = np.ascontiguousarray(Xq, dtype=np.int8)
        CB = np.ascontiguousarray(CB, dtype=np.int8)
        T, K = Xq.shape
        N = CB.shape[0]
        if CB.shape[1] != K:
            raise ValueError("int8_matmul: inner dimensions differ")
        assert K * Q_MAX * Q_MAX < 2**31, "int32 accumulator would overflow"
        acc = np.empty((T, N), np.int32)
        self.lib.oref_int8_matmul(_p(Xq), T, K, _p(CB), N, _p(acc), self.threads)
        return acc

    def _combine(self, acc, sA, SCB, Xo16, Wo16, bias16, elem: int) -> np.ndarray:
        acc = np.ascontiguousarray(acc, dtype=np.int32)
        sA = np.ascontiguousarray(sA, dtype=np.float32)
        SCB = np.ascontiguousarray(SCB, dtype=np.float32)
        Xo16 = np.ascontiguousarray(Xo16, dtype=np.uint16)
        Wo16 = np.ascontiguousarray(Wo16, dtype=np.uint16)
        T, N = acc.shape
        n = Xo16.shape[1]
        b = None if bias16 is None else np.ascontiguousarray(bias16, dtype=np.uint16)
        Y = np.empty((T, N), np.float64)
        self.lib.oref_combine(_p(acc), _p(sA), _p(SCB), _p(Xo16), _p(Wo16), n, _p(b), elem, T, N, _p(Y),
                              self.threads)
        return Y

    # -- fp16 API of the numpy oracle -------------------------------------------
    @staticmethod
    def _u16(a):
        return np.ascontiguousarray(a, dtype=np.float16).view(np.uint16)

    def quantize_weight(self, W):
        return self._quantize_weight(self._u16(W), F16)

    def outlier_mask(self, X, threshold):
        return self._mask(self._u16(X), threshold, F16)

    def quantize_rows(self, X, mask):
        return self._rows(self._u16(X), mask, F16)

    def outlier_operands(self, X, CB, SCB, idx):
        Xo, Wo = self._operands(self._u16(X), CB, SCB, idx, F16)
        return Xo.view(np.float16), Wo.view(np.float16)

    def combine(self, acc, sA, SCB, Xo, Wo, bias):
        return self._combine(acc, sA, SCB, self._u16(Xo), self._u16(Wo), None if bias is None else self._u16(bias),
                             F16)

    def _forward16(self, X16, CB, SCB, bias16, threshold, rows, elem, Wo16_from=None):
        X16 = np.ascontiguousarray(X16, dtype=np.uint16)
        mask = self._mask(X16, threshold, elem)
        idx = self.outlier_index(mask)
        Xs = X16 if rows is None else np.ascontiguousarray(X16[np.asarray(rows)])
        Xq, sA = self._rows(Xs, mask, elem)
        Xo, Wo = self._operands(Xs, CB, SCB, idx, elem)
        if Wo16_from is not None:  # has_fp16_weights=True: the 16-bit weight's own columns
            Wo = np.ascontiguousarray(Wo16_from[:, idx])
        acc = self.int8_matmul(Xq, CB)
        Y = self._combine(acc, sA, SCB, Xo, Wo, bias16, elem)
        return {"mask": mask, "idx": idx, "n_out": int(idx.size), "Xq": Xq, "sA": sA, "Xo": Xo, "Wo": Wo,
                "acc": acc, "Y": Y}

    def linear_forward(self, X, CB, SCB, bias, threshold, rows=None) -> dict:
        r = self._forward16(self._u16(X), CB, SCB, None if bias is None else self._u16(bias), threshold, rows, F16)
        r["Xo"], r["Wo"] = r["Xo"].view(np.float16), r["Wo"].view(np.float16)
        return r

    def linear_forward_fp16w(self, X, W, bias, threshold, rows=None) -> dict:
        W16 = self._u16(W)
        CB, SCB = self._quantize_weight(W16, F16)
        r = self._forward16(self._u16(X), CB, SCB, None if bias is None else self._u16(bias), threshold, rows, F16,
                            Wo16_from=W16)
        r["Xo"], r["Wo"] = r["Xo"].view(np.float16), r["Wo"].view(np.float16)
        r["CB"], r["SCB"] = CB, SCB
        return r

    # -- bf16 API (bit patterns in and out) ---------------------------------------
    def quantize_weight_bf16(self, W_u16):
        return self._quantize_weight(W_u16, BF16)

    def linear_forward_bf16(self, X_u16, CB, SCB, bias_u16, threshold, rows=None) -> dict:
        return self._forward16(X_u16, CB, SCB, bias_u16, threshold, rows, BF16)

    def linear_forward_fp16w_bf16(self, X_u16, W_u16, bias_u16, threshold, rows=None) -> dict:
        W16 = np.ascontiguousarray(W_u16, dtype=np.uint16)
        CB, SCB = self._quantize_weight(W16, BF16)
        r = self._forward16(X_u16, CB, SCB, bias_u16, threshold, rows, BF16, Wo16_from=W16)
        r["CB"], r["SCB"] = CB, SCB
        return r

    # -- the stated tolerances of a 16-bit Y -----------------------------------------
    @staticmethod
    def y_tolerance(Yref) -> float:
        return 1e-3 * float(np.abs(Yref).max(initial=0.0)) + 2e-3

    @staticmethod
    def y_tolerance_bf16(Yref) -> float:
        return 2.0**-8 * float(np.abs(Yref).max(initial=0.0)) + 2e-3


_default: Oracle | None = None


def default() -> Oracle:
    """The C++ oracle built from ``llm_int8_ref.cpp`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
