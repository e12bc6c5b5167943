"""The C-ABI library loads and exports what include/*.h declares; host-only logic.

No CUDA call is made here: these run on machines without a GPU.
"""

from __future__ import annotations

import ctypes
import glob
import os
import re

import numpy as np
import pytest

from int8_mixed_precision_column_b200 import build, native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return native.lib()


def declared_functions() -> list[str]:
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(int8_\w+)\s*\(", src, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("int8_quantize_weight", "int8_linear_forward", "int8_linear_workspace_bytes",
                 "int8_check_status", "int8_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(names) <= set(native.SIGNATURES), "binding lacks a signature for a declared entry point"


def test_status_strings(lib):
    assert native.int8_status_string(0) == "I8_OK"
    assert native.int8_status_string(4) == "I8_ERR_TIMEOUT"
    assert native.int8_status_string(99) == "I8_ERR_UNKNOWN"
    assert lib.int8_version() >= 100


def _half_values():
    bits = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    return bits, bits.view(np.float16).astype(np.float32)


@pytest.mark.parametrize("thr", [6.0, 0.1, 1e-8, 3.14159, 65504.0, 70000.0, 6.000001, float("inf")])
def test_threshold_bits_match_fp32_comparison(lib, thr):
    """(bits & 0x7fff) > H and not NaN  <=>  |float(x)| > float32(thr), for every fp16 x."""
    H = native.int8_outlier_threshold_bits(thr)
    bits, vals = _half_values()
    mag = bits.astype(np.uint32) & 0x7FFF
    kernel_rule = (mag > H) & (mag <= 0x7C00)
    with np.errstate(invalid="ignore"):
        fp32_rule = np.abs(vals) > np.float32(thr)
    assert np.array_equal(kernel_rule, fp32_rule)


@pytest.mark.parametrize("thr", [0.0, -1.0, float("nan")])
def test_threshold_off(lib, thr):
    assert native.int8_outlier_threshold_bits(thr) == 0xFFFFFFFF


def test_workspace_layout(lib):
    T, K, N = 100, 208, 272
    L = native.int8_linear_workspace_layout(T, K, N)
    assert L["ldo"] == 256
    assert L["status"] == 0 and L["mask"] >= 64
    offs = [L["mask"], L["sA"], L["Xq"], L["Xo"], L["Wo"], L["total"]]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert L["sA"] >= L["mask"] + (K + 31) // 32 * 4
    assert L["Xo"] >= L["Xq"] + T * K
    assert L["Wo"] >= L["Xo"] + T * L["ldo"] * 2
    assert L["total"] >= L["Wo"] + N * L["ldo"] * 2
    assert native.int8_linear_workspace_bytes(T, K, N) == L["total"]
    assert native.int8_linear_forward_host_workspace_bytes(T, K, N) >= L["total"] + T * K * 2 + T * N * 2


@pytest.mark.parametrize("T,K,N", [(4, 15, 64), (4, 64, 8), (-1, 64, 64), (4, 0, 64), (4, 131088, 64)])
def test_bad_shapes_rejected_before_any_cuda_call(lib, T, K, N):
    assert native.int8_linear_workspace_bytes(T, K, N) == 0
    st = lib.int8_linear_forward(None, T, K, None, None, None, N, 6.0, None, None, None, None, 0, None)
    assert st == 1  # I8_ERR_INVALID_ARG
    st = lib.int8_quantize_weight(None, N, K, None, None, None)
    assert st == 1


def test_null_pointers_rejected(lib):
    st = lib.int8_linear_forward(None, 4, 64, None, None, None, 64, 6.0, None, None, None, None, 0, None)
    assert st == 1
    assert lib.int8_check_status(None, None, None) == 2  # I8_ERR_WORKSPACE


def test_small_workspace_rejected(lib):
    # all pointers non-null and aligned (never dereferenced: validation fails first)
    fake = ctypes.c_void_p(1 << 20)
    st = lib.int8_linear_forward(fake, 4, 64, fake, fake, None, 64, 6.0, fake, fake, fake, fake, 16, None)
    assert st == 2  # I8_ERR_WORKSPACE


@pytest.mark.parametrize("which,offset", [("X", 8), ("CB", 8), ("Y", 8), ("SCB", 2), ("idx", 2), ("n_out", 2),
                                          ("bias", 1), ("ws", 128)])
def test_misaligned_pointers_rejected_before_any_cuda_call(lib, which, offset):
    # X, CB and Y need 16-byte alignment (16-byte vector and TMA accesses), SCB,
    # idx and n_out 4, the bias 2, the workspace 256 (its carve-outs); the
    # addresses are never dereferenced: validation fails first
    T, K, N = 4, 64, 64
    ws_bytes = native.int8_linear_workspace_bytes(T, K, N)
    ptr = {k: 1 << 20 for k in ("X", "CB", "SCB", "bias", "Y", "idx", "n_out", "ws")}
    ptr[which] += offset
    v = {k: ctypes.c_void_p(a) for k, a in ptr.items()}
    st = lib.int8_linear_forward(v["X"], T, K, v["CB"], v["SCB"], v["bias"], N, 6.0, v["Y"], v["idx"], v["n_out"],
                                 v["ws"], ws_bytes, None)
    assert st == (2 if which == "ws" else 1)  # I8_ERR_WORKSPACE / I8_ERR_INVALID_ARG


def _bf16_values():
    bits = np.arange(0, 0x10000, dtype=np.uint32)
    return bits, (bits << 16).view(np.float32)


@pytest.mark.parametrize("thr", [6.0, 0.1, 1e-8, 3.14159, 6.000001, 6.03125, 3.0e38, 3.4e38, float("inf"), 1e-40])
def test_bf16_threshold_bits_match_fp32_comparison(lib, thr):
    """bf16: (bits & 0x7fff) > H and not NaN  <=>  |float(x)| > float32(thr), for every bf16 x."""
    H = native.int8_outlier_threshold_bits(thr, native.torch.bfloat16)
    bits, vals = _bf16_values()
    mag = bits & 0x7FFF
    kernel_rule = (mag > H) & (mag <= 0x7F80)
    with np.errstate(invalid="ignore"):
        fp32_rule = np.abs(vals) > np.float32(thr)
    assert np.array_equal(kernel_rule, fp32_rule)


@pytest.mark.parametrize("thr", [0.0, -1.0, float("nan")])
def test_bf16_threshold_off(lib, thr):
    assert lib.int8_outlier_threshold_bits_ex(thr, native.I8_DTYPE_BF16) == 0xFFFFFFFF


def test_unknown_dtype_rejected_before_any_cuda_call(lib):
    assert lib.int8_outlier_threshold_bits_ex(6.0, 2) == 0xFFFFFFFE
    fake = ctypes.c_void_p(1 << 20)
    big = native.int8_linear_workspace_bytes(4, 64, 64)
    for dt in (-1, 2, 7):
        st = lib.int8_linear_forward_ex(fake, dt, 4, 64, fake, fake, None, 64, 6.0, fake, fake, fake, fake, big, 0,
                                        None, None)
        assert st == 1
        assert lib.int8_quantize_weight_ex(fake, dt, 64, 64, fake, fake, None) == 1
        st = lib.int8_linear_forward_fp16w_ex(fake, dt, 4, 64, fake, None, 64, 6.0, fake, fake, fake, fake, 1 << 30,
                                              None)
        assert st == 1
