"""The forward that needs no scratch allocation (int8_linear_forward_decode_static).

It serves callers that can neither allocate device memory nor pass a
workspace (e.g. a plugin whose host runtime forbids allocation inside its
execute call, or an application held to a fixed device-memory budget).  Its
scratch is a fixed array inside the library, shared by every call and keeping
the previous call's contents.  Three calls in a row -- 40 planted outlier
columns, then 2, then none at all (threshold 0) -- are each compared with the
workspace-based int8_linear_forward on the same inputs, bit for bit (the same
kernels run on both paths, so a read of stale scratch left by the previous
call would show up as a difference), and with the CPU oracle at the stated
fp16 tolerance.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from oracle import llm_int8 as O
from int8_mixed_precision_column_b200 import build, native, workloads

pytestmark = pytest.mark.gpu


def static_forward(X, CB, SCB, bias, threshold):
    T, K = X.shape
    N = CB.shape[0]
    Y = torch.empty((T, N), dtype=torch.float16, device="cuda")
    idx = torch.full((K,), -1, dtype=torch.int32, device="cuda")
    n_out = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = native.lib().int8_linear_forward_decode_static(
        X.data_ptr(), T, K, CB.data_ptr(), SCB.data_ptr(), None if bias is None else bias.data_ptr(), N,
        float(threshold), Y.data_ptr(), idx.data_ptr(), n_out.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    return st, Y, idx, n_out


def test_static_scratch_forward_matches_workspace_forward_and_oracle():
    assert torch.cuda.is_available()
    build.build()
    native.lib()
    problems = [
        workloads.make_problem("first", 16, 4096, 1024, n_planted=40, bias_std=0.01, seed=21),
        workloads.make_problem("second", 3, 4096, 1024, n_planted=2, bias_std=0.01, seed=22),
        workloads.make_problem("third", 16, 4096, 1024, n_planted=40, bias_std=0.01, threshold=0.0, seed=23),
    ]
    for p in problems:
        X, W, b = p.X.cuda(), p.W.cuda(), p.bias.cuda()
        CB, SCB = native.int8_quantize_weight(W)
        st, Y, idx, n_out = static_forward(X, CB, SCB, b, p.threshold)
        assert st == 0, f"{native.int8_status_string(st)} ({native.int8_last_cuda_error()})"
        Yr, idxr, nr, ws = native.int8_linear_forward(X, CB, SCB, b, p.threshold)
        assert native.int8_check_status(ws)[0] == 0
        torch.cuda.synchronize()
        n = int(nr.item())
        assert int(n_out.item()) == n
        assert n == 0 if p.threshold <= 0 else n >= len(p.planted_cols)
        assert torch.equal(idx[:n], idxr[:n])
        assert torch.equal(Y.view(torch.int16), Yr.view(torch.int16)), p.name
        # the oracle, from the fp16 weight (nothing it consumes comes from the GPU)
        CBo, SCBo = O.quantize_weight(p.W.numpy())
        r = O.linear_forward(p.X.numpy(), CBo, SCBo, p.bias.numpy(), p.threshold)
        assert n == r["n_out"] and np.array_equal(idx[:n].cpu().numpy(), r["idx"])
        err = np.abs(Y.cpu().numpy().astype(np.float64) - r["Y"]).max()
        assert err <= O.y_tolerance(r["Y"]), (p.name, err)


def test_static_scratch_rejects_sizes_beyond_its_capacity():
    build.build()
    lib = native.lib()
    fake = ctypes.c_void_p(1 << 20)
    # T = 16, K = 87424 needs more than the 4 MiB scratch: refused before any work
    assert lib.int8_linear_forward_decode_static(fake, 16, 87424, fake, fake, None, 64, 6.0, fake, fake, fake,
                                                 None) == 2  # I8_ERR_WORKSPACE
    # more than 16 tokens is not the decode case
    assert lib.int8_linear_forward_decode_static(fake, 17, 64, fake, fake, None, 64, 6.0, fake, fake, fake,
                                                 None) == 1  # I8_ERR_INVALID_ARG
