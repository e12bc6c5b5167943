"""has_fp16_weights=True forward (int8_linear_forward_fp16w) against the oracle."""

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


def _u256(v):
    return (v + 255) // 256 * 256


@pytest.mark.parametrize("T,K,N,planted,thr", [(16, 1024, 512, 5, 6.0), (200, 1024, 528, 9, 6.0),
                                               (5, 256, 96, 3, 0.0), (40, 512, 256, 70, 6.0), (16, 128, 64, 0, 0.1)])
def test_fp16w_forward_matches_oracle(T, K, N, planted, thr):
    p = workloads.make_problem("fp16w", T, K, N, n_planted=planted, bias_std=0.01, threshold=thr, seed=T + K)
    X = p.X
    if thr == 0.1:
        X[X.abs() <= 0.1] = 0.5
    Y, idx, n_out, ws = native.int8_linear_forward_fp16w(X.cuda(), p.W.cuda(), p.bias.cuda(), thr)
    st, where = native.int8_check_status(ws)
    assert st == 0, f"device status {st} at {where:#x} ({native.int8_last_cuda_error()})"
    r = O.linear_forward_fp16w(X.numpy(), p.W.numpy(), p.bias.numpy(), thr)
    n = int(n_out.item())
    assert n == r["n_out"] and np.array_equal(idx[:n].cpu().numpy(), r["idx"])
    L = native.int8_linear_workspace_layout(T, K, N)
    cb = ws[L["total"]: L["total"] + N * K].view(torch.int8).view(N, K).cpu().numpy()
    so = _u256(L["total"] + N * K)
    scb = ws[so: so + 4 * N].view(torch.float32).cpu().numpy()
    assert np.array_equal(cb, r["CB"]) and np.array_equal(scb, r["SCB"])
    v = native.workspace_views(ws, T, K, N)
    assert np.array_equal(v["Xq"].cpu().numpy(), r["Xq"]) and np.array_equal(v["sA"].cpu().numpy(), r["sA"])
    if n and T > 16:
        assert np.array_equal(v["Wo"][:, :n].cpu().numpy(), r["Wo"])
    err = np.abs(Y.cpu().numpy().astype(np.float64) - r["Y"]).max()
    assert err <= O.y_tolerance(r["Y"])
