"""Guard regions around every buffer the library writes.

compute-sanitizer is not available here, so out-of-bounds writes are caught
with canaries instead.  Each caller-owned output (CB, SCB, Y, idx, n_out) and
the workspace is carved out of a larger allocation whose bytes before and
after it (4 KB each side) hold a canary pattern, and so does the buffer
itself before the call (the library may not rely on its contents).  After
the call every guard byte must be intact, and the outputs must equal, bit for
bit, those of the same call on plain buffers (the forward is deterministic).
"""
from __future__ import annotations

import pytest
import torch

from int8_mixed_precision_column_b200 import build, native, workloads

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    native.lib()


class Guarded:
    """`nbytes` of device memory between two canary-filled guard regions."""

    def __init__(self, nbytes: int):
        self.n = int(nbytes)
        self.buf = torch.full((GUARD + self.n + GUARD,), CANARY, dtype=torch.uint8, device="cuda")

    def view(self, dtype: torch.dtype, shape) -> torch.Tensor:
        return self.buf[GUARD:GUARD + self.n].view(dtype).view(shape)

    def bytes(self) -> torch.Tensor:
        return self.buf[GUARD:GUARD + self.n]

    def intact(self) -> bool:
        return bool((self.buf[:GUARD] == CANARY).all()) and bool((self.buf[GUARD + self.n:] == CANARY).all())


def _esize(dtype: torch.dtype) -> int:
    return torch.tensor([], dtype=dtype).element_size()


FORWARD_CASES = [
    # T, K, N, planted, threshold, path, dtype
    (1, 1040, 336, 3, 6.0, native.PATH_AUTO, torch.float16),            # decode GEMV, one-kernel prep
    (16, 2048, 528, 9, 6.0, native.PATH_DECODE, torch.bfloat16),        # decode, cluster-form prep
    (5, 20480, 96, 4, 6.0, native.PATH_DECODE, torch.float16),          # decode, rows not held in registers
    (200, 208, 272, 3, 6.0, native.PATH_TENSOR_CORE, torch.float16),    # pair GEMM, ragged
    (300, 336, 784, 70, 6.0, native.PATH_TENSOR_CORE, torch.bfloat16),  # two outlier K-blocks
    (130, 1024, 528, 17, 6.0, native.PATH_TENSOR_CORE_1SM, torch.float16),
    (1100, 336, 8208, 70, 6.0, native.PATH_TENSOR_CORE, torch.float16),  # more tiles than SM pairs
    (64, 256, 96, 4, 0.0, native.PATH_AUTO, torch.float16),             # decomposition off
    (40, 128, 64, 0, 0.1, native.PATH_TENSOR_CORE, torch.float16),      # every column an outlier
]


@pytest.mark.parametrize("T,K,N,planted,thr,path,dtype", FORWARD_CASES)
def test_forward_writes_stay_inside_their_buffers(T, K, N, planted, thr, path, dtype):
    p = workloads.make_problem("guard", T, K, N, n_planted=planted, bias_std=0.01, threshold=thr,
                               seed=T + K + N, device="cuda")
    X, W, b = p.X.to(dtype), p.W.to(dtype), p.bias.to(dtype)

    # weight quantisation into guarded CB / SCB
    gCB, gSCB = Guarded(N * K), Guarded(N * 4)
    CB, SCB = native.int8_quantize_weight(W, CB=gCB.view(torch.int8, (N, K)), SCB=gSCB.view(torch.float32, (N,)))
    CB_ref, SCB_ref = native.int8_quantize_weight(W)
    torch.cuda.synchronize()
    assert gCB.intact() and gSCB.intact()
    assert torch.equal(CB, CB_ref) and torch.equal(SCB, SCB_ref)

    # the forward into guarded Y / idx / n_out / workspace
    gY = Guarded(T * N * _esize(dtype))
    gidx, gn = Guarded(K * 4), Guarded(4)
    gws = Guarded(native.int8_linear_workspace_bytes(T, K, N))
    Y, idx, n_out, ws = native.int8_linear_forward(
        X, CB, SCB, b, thr, Y=gY.view(dtype, (T, N)), idx=gidx.view(torch.int32, (K,)),
        n_out=gn.view(torch.int32, (1,)), workspace=gws.bytes(), path=path)
    st, where = native.int8_check_status(ws)
    assert st == 0, f"device status {st} at {where:#x}"
    Y_ref, idx_ref, n_ref, _ = native.int8_linear_forward(X, CB_ref, SCB_ref, b, thr, path=path)
    torch.cuda.synchronize()
    for name, g in (("Y", gY), ("idx", gidx), ("n_out", gn), ("workspace", gws)):
        assert g.intact(), f"a write outside {name}"
    n = int(n_out.item())
    assert n == int(n_ref.item())
    assert torch.equal(idx[:n], idx_ref[:n])
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))


@pytest.mark.parametrize("T,K,N,planted", [(16, 1024, 512, 5), (200, 1024, 528, 9)])
def test_fp16w_forward_writes_stay_inside_their_buffers(T, K, N, planted):
    p = workloads.make_problem("guardw", T, K, N, n_planted=planted, bias_std=0.01, seed=T + N, device="cuda")
    gY = Guarded(T * N * 2)
    gidx, gn = Guarded(K * 4), Guarded(4)
    gws = Guarded(native.lib().int8_linear_fp16w_workspace_bytes(T, K, N))
    Y, idx, n_out, ws = native.int8_linear_forward_fp16w(
        p.X, p.W, p.bias, p.threshold, Y=gY.view(torch.float16, (T, N)), idx=gidx.view(torch.int32, (K,)),
        n_out=gn.view(torch.int32, (1,)), workspace=gws.bytes())
    Y_ref, idx_ref, n_ref, _ = native.int8_linear_forward_fp16w(p.X, p.W, p.bias, p.threshold)
    torch.cuda.synchronize()
    for name, g in (("Y", gY), ("idx", gidx), ("n_out", gn), ("workspace", gws)):
        assert g.intact(), f"a write outside {name}"
    n = int(n_out.item())
    assert n == int(n_ref.item()) and torch.equal(idx[:n], idx_ref[:n])
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
