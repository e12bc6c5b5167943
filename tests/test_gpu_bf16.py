"""bf16 element type (int8_quantize_weight_ex / int8_linear_forward_ex /
int8_linear_forward_fp16w_ex) against the oracle's bf16 forward.

The integer stages (CB, SCB, idx, n_out, Xq, sA) and the gathered outlier
operands (Xo, Wo as bf16 patterns) are compared bit for bit; Y within the
bf16 output bound 2^-8 max|Yref| + 2e-3.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import llm_int8 as O
from int8_mixed_precision_column_b200 import build, native, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available()
    build.build()
    native.lib()


def _u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> its bit patterns (uint16)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16_problem(T, K, N, planted, thr, seed, bias=True):
    p = workloads.make_problem("bf16", T, K, N, n_planted=planted, bias_std=0.01 if bias else None,
                               threshold=thr, seed=seed)
    X = p.X.to(torch.bfloat16)
    W = p.W.to(torch.bfloat16)
    b = p.bias.to(torch.bfloat16) if bias else None
    return X, W, b


def _check_stages(ws, T, K, N, n, r, check_wo):
    v = native.workspace_views(ws, T, K, N, torch.bfloat16)
    assert np.array_equal(v["Xq"].cpu().numpy(), r["Xq"])
    assert np.array_equal(v["sA"].cpu().numpy(), r["sA"])
    if n:
        assert np.array_equal(_u16(v["Xo"][:, :n]), r["Xo"])
        assert np.all(_u16(v["Xo"][:, n: (n + 63) // 64 * 64]) == 0)
        if check_wo:
            assert np.array_equal(_u16(v["Wo"][:, :n]), r["Wo"])


def test_bf16_quantize_weight_bit_exact():
    _, W, _ = _bf16_problem(4, 1040, 336, 0, 6.0, seed=3)
    W[5, 7] = 0.0
    W[9] = 0.0                      # an all-zero row: SCB 0, codes 0
    CB, SCB = native.int8_quantize_weight(W.cuda())
    cb, scb = O.quantize_weight_bf16(_u16(W))
    assert np.array_equal(CB.cpu().numpy(), cb) and np.array_equal(SCB.cpu().numpy(), scb)


@pytest.mark.parametrize("path", [native.PATH_AUTO, native.PATH_TENSOR_CORE, native.PATH_TENSOR_CORE_1SM,
                                  native.PATH_DECODE])
@pytest.mark.parametrize("T,K,N,planted,thr", [(1, 1024, 512, 3, 6.0), (16, 2048, 528, 7, 6.0),
                                               (9, 256, 96, 0, 0.0), (200, 1024, 528, 9, 6.0),
                                               (300, 512, 784, 70, 6.0), (130, 4096, 256, 200, 6.0)])
def test_bf16_forward_matches_oracle(path, T, K, N, planted, thr):
    if path == native.PATH_DECODE and T > native.DECODE_MAX_T:
        pytest.skip("decode path takes T <= 16")
    X, W, b = _bf16_problem(T, K, N, planted, thr, seed=T * 7 + K + N)
    CB, SCB = native.int8_quantize_weight(W.cuda())
    Y, idx, n_out, ws = native.int8_linear_forward(X.cuda(), CB, SCB, b.cuda(), thr, path=path)
    st, where = native.int8_check_status(ws)
    assert st == 0, f"device status {st} at {where:#x} ({native.int8_last_cuda_error()})"
    assert Y.dtype == torch.bfloat16
    r = O.linear_forward_bf16(_u16(X), CB.cpu().numpy(), SCB.cpu().numpy(), _u16(b), thr)
    n = int(n_out.item())
    assert n == r["n_out"] and np.array_equal(idx[:n].cpu().numpy(), r["idx"])
    gemv = path == native.PATH_DECODE or (path == native.PATH_AUTO and T <= native.DECODE_MAX_T)
    _check_stages(ws, T, K, N, n, r, check_wo=not gemv)
    err = np.abs(Y.float().cpu().numpy().astype(np.float64) - r["Y"]).max()
    assert err <= O.y_tolerance_bf16(r["Y"]), err


def test_bf16_pair_tiles_outnumber_pairs():
    """bf16 through the SM-pair kernel with 85 output tiles for 74 pairs, two
    outlier K-blocks and ragged last tiles; sampled rows, every column."""
    T, K, N = 1100, 336, 8208
    X, W, b = _bf16_problem(T, K, N, 70, 6.0, seed=5)
    CB, SCB = native.int8_quantize_weight(W.cuda())
    Y, idx, n_out, ws = native.int8_linear_forward(X.cuda(), CB, SCB, b.cuda(), 6.0, path=native.PATH_TENSOR_CORE)
    st, where = native.int8_check_status(ws)
    assert st == 0, f"device status {st} at {where:#x} ({native.int8_last_cuda_error()})"
    rows = list(range(0, T, 37)) + [T - 1]
    r = O.linear_forward_bf16(_u16(X), CB.cpu().numpy(), SCB.cpu().numpy(), _u16(b), 6.0, rows=rows)
    n = int(n_out.item())
    assert n == r["n_out"] > 64 and np.array_equal(idx[:n].cpu().numpy(), r["idx"])
    v = native.workspace_views(ws, T, K, N, torch.bfloat16)
    rt = torch.as_tensor(rows, device="cuda")
    assert np.array_equal(v["Xq"][rt].cpu().numpy(), r["Xq"])
    assert np.array_equal(v["sA"][rt].cpu().numpy(), r["sA"])
    err = np.abs(Y[rt].float().cpu().numpy().astype(np.float64) - r["Y"]).max()
    assert err <= O.y_tolerance_bf16(r["Y"]), err


def test_bf16_no_bias_and_every_column_flagged():
    T, K, N = 24, 128, 64
    X, W, _ = _bf16_problem(T, K, N, 0, 0.0, seed=11, bias=False)
    X[X.abs() < 0.5] = 0.75
    CB, SCB = native.int8_quantize_weight(W.cuda())
    Y, idx, n_out, ws = native.int8_linear_forward(X.cuda(), CB, SCB, None, 0.1, path=native.PATH_TENSOR_CORE)
    assert native.int8_check_status(ws)[0] == 0
    r = O.linear_forward_bf16(_u16(X), CB.cpu().numpy(), SCB.cpu().numpy(), None, 0.1)
    assert int(n_out.item()) == K == r["n_out"]
    _check_stages(ws, T, K, N, K, r, check_wo=True)
    err = np.abs(Y.float().cpu().numpy().astype(np.float64) - r["Y"]).max()
    assert err <= O.y_tolerance_bf16(r["Y"])


@pytest.mark.parametrize("T,K,N,planted,thr", [(16, 1024, 512, 5, 6.0), (200, 1024, 528, 9, 6.0),
                                               (40, 512, 256, 70, 6.0)])
def test_bf16_fp16w_forward_matches_oracle(T, K, N, planted, thr):
    X, W, b = _bf16_problem(T, K, N, planted, thr, seed=T + K + 1)
    Y, idx, n_out, ws = native.int8_linear_forward_fp16w(X.cuda(), W.cuda(), b.cuda(), thr)
    st, where = native.int8_check_status(ws)
    assert st == 0, f"device status {st} at {where:#x} ({native.int8_last_cuda_error()})"
    r = O.linear_forward_fp16w_bf16(_u16(X), _u16(W), _u16(b), thr)
    n = int(n_out.item())
    assert n == r["n_out"] and np.array_equal(idx[:n].cpu().numpy(), r["idx"])
    _check_stages(ws, T, K, N, n, r, check_wo=T > native.DECODE_MAX_T)
    err = np.abs(Y.float().cpu().numpy().astype(np.float64) - r["Y"]).max()
    assert err <= O.y_tolerance_bf16(r["Y"]), err


def test_bf16_llama_width_prefill_sampled_rows():
    """The Llama-7B-width prefill (2048 x 4096 -> 4096) in bf16 on the default
    path; the oracle checks a sample of rows (integer stages for all rows)."""
    p = workloads.llama7b_prefill(seed=5)
    X = p.X.to(torch.bfloat16)
    W = p.W.to(torch.bfloat16)
    b = p.bias.to(torch.bfloat16)
    CB, SCB = native.int8_quantize_weight(W.cuda())
    Y, idx, n_out, ws = native.int8_linear_forward(X.cuda(), CB, SCB, b.cuda(), 6.0)
    assert native.int8_check_status(ws)[0] == 0
    rows = np.array([0, 1, 127, 128, 1000, 2047])
    r = O.linear_forward_bf16(_u16(X), CB.cpu().numpy(), SCB.cpu().numpy(), _u16(b), 6.0, rows=rows)
    n = int(n_out.item())
    assert n == r["n_out"] and np.array_equal(idx[:n].cpu().numpy(), r["idx"])
    v = native.workspace_views(ws, 2048, 4096, 4096, torch.bfloat16)
    assert np.array_equal(v["Xq"][rows].cpu().numpy(), r["Xq"])
    assert np.array_equal(v["sA"][rows].cpu().numpy(), r["sA"])
    err = np.abs(Y[rows].float().cpu().numpy().astype(np.float64) - r["Y"]).max()
    assert err <= O.y_tolerance_bf16(r["Y"]), err
