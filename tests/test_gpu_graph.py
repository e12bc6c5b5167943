"""A forward captured once in a CUDA graph and replayed (the way a serving
loop runs a layer) gives the eager forward's outputs bit for bit, also after
new activations are copied into the captured input buffer."""

from __future__ import annotations

import pytest
import torch

from int8_mixed_precision_column_b200 import build, native, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available()
    build.build()
    native.lib()


@pytest.mark.parametrize("T,K,N,path", [(8, 1024, 512, native.PATH_AUTO), (256, 2048, 1024, native.PATH_AUTO),
                                        (200, 1024, 528, native.PATH_TENSOR_CORE_1SM)])
def test_forward_replays_from_a_cuda_graph(T, K, N, path):
    p = workloads.make_problem("graph", T, K, N, n_planted=5, bias_std=0.01, seed=T + K, device="cuda")
    q = workloads.make_problem("graph2", T, K, N, n_planted=9, bias_std=0.01, seed=T + K + 1, device="cuda")
    CB, SCB = native.int8_quantize_weight(p.W)
    X = p.X.clone()
    Y = torch.empty((T, N), dtype=torch.float16, device="cuda")
    idx = torch.empty((K,), dtype=torch.int32, device="cuda")
    n_out = torch.empty((1,), dtype=torch.int32, device="cuda")
    ws = native.new_workspace(T, K, N)

    def fwd():
        native.int8_linear_forward(X, CB, SCB, p.bias, p.threshold, Y=Y, idx=idx, n_out=n_out, workspace=ws,
                                   path=path)

    refs = []
    for Xin in (p.X, q.X):
        Yr, idxr, nr, wsr = native.int8_linear_forward(Xin, CB, SCB, p.bias, p.threshold, path=path)
        assert native.int8_check_status(wsr)[0] == 0
        refs.append((Yr.clone(), idxr[: int(nr.item())].clone()))

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fwd()  # warm-up outside the capture (one-time attribute and occupancy queries)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    for Xin, (Yr, idxr) in zip((p.X, q.X, p.X), (refs[0], refs[1], refs[0])):
        X.copy_(Xin)
        Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert native.int8_check_status(ws)[0] == 0
        assert int(n_out.item()) == idxr.numel() and torch.equal(idx[: idxr.numel()], idxr)
        assert torch.equal(Y.view(torch.int16), Yr.view(torch.int16))
    del g
