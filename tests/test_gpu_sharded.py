"""N-sharded forward on one GPU (int8_linear_forward_sharded, sharded.py).

The g ranks of an N-sharded layer are emulated one after another on one GPU,
with no rank waiting on another: rank r runs its shard with the g output
buffers as destinations (its own first), exactly as it would store into the
peers' buffers on g GPUs.  Afterwards every buffer must hold the unsharded
forward's Y bit for bit (each output element is computed by the same
arithmetic whichever shard it falls in), and every buffer is compared with
the CPU oracle's forward of the whole layer at the stated tolerance (fp16:
1e-3 max|Yref| + 2e-3; bf16: 2^-8 max|Yref| + 2e-3).  A world-size-1 process
group checks the torch plumbing of both assembly modes, also against the
oracle.
"""

from __future__ import annotations

import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from oracle import llm_int8 as O
from int8_mixed_precision_column_b200 import build, native, sharded, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available()
    build.build()
    native.lib()


def _layer(T, K, N, planted, dtype, seed, with_oracle=False):
    p = workloads.make_problem("shard", T, K, N, n_planted=planted, bias_std=0.01, seed=seed, device="cuda")
    X, W, b = p.X.to(dtype), p.W.to(dtype), p.bias.to(dtype)
    CB, SCB = native.int8_quantize_weight(W)
    if not with_oracle:
        return X, CB, SCB, b
    return X, CB, SCB, b, _oracle(X, W, b, 6.0)


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle(X, W, b, thr):
    """The oracle's forward of the whole (unsharded) layer, from the 16-bit
    X, W and bias; returns (Yref fp64, tolerance)."""
    if X.dtype == torch.bfloat16:
        CBo, SCBo = O.quantize_weight_bf16(_u16(W))
        r = O.linear_forward_bf16(_u16(X), CBo, SCBo, _u16(b), thr)
        return r, O.y_tolerance_bf16(r["Y"])
    CBo, SCBo = O.quantize_weight(W.cpu().numpy())
    r = O.linear_forward(X.cpu().numpy(), CBo, SCBo, b.cpu().numpy(), thr)
    return r, O.y_tolerance(r["Y"])


def _check_oracle(Y, ref):
    r, tol = ref
    err = np.abs(Y.float().cpu().numpy().astype(np.float64) - r["Y"]).max(initial=0.0)
    assert err <= tol, f"max|Y-Yref| = {err:.3g} > {tol:.3g}"


def _bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("T,K,N,world,path", [
    (200, 1024, 1024, 2, native.PATH_TENSOR_CORE),
    (300, 512, 784, 3, native.PATH_TENSOR_CORE),
    (130, 2048, 4096, 8, native.PATH_TENSOR_CORE_1SM),
    (16, 2048, 2048, 4, native.PATH_DECODE),
    (5, 1024, 1040, 5, native.PATH_AUTO),
])
def test_emulated_ranks_fill_every_buffer_with_the_unsharded_output(dtype, T, K, N, world, path):
    X, CB, SCB, b, ref = _layer(T, K, N, 6, dtype, seed=T + N + world, with_oracle=True)
    Y_ref, idx_ref, n_ref, ws_ref = native.int8_linear_forward(X, CB, SCB, b, 6.0, path=path)
    assert native.int8_check_status(ws_ref)[0] == 0
    n = int(n_ref.item())
    bufs = [torch.full((T, N), float("nan"), dtype=dtype, device="cuda") for _ in range(world)]
    for r in range(world):
        CBs, SCBs, bs, lo, hi = sharded.shard_layer(CB, SCB, b, world, r)
        dst = [bufs[r]] + [bufs[q] for q in range(world) if q != r]
        idx, n_out, ws = native.int8_linear_forward_sharded(X, CBs, SCBs, bs, 6.0, dst, N, lo, path=path)
        st, where = native.int8_check_status(ws)
        assert st == 0, f"device status {st} at {where:#x} ({native.int8_last_cuda_error()})"
        assert int(n_out.item()) == n and torch.equal(idx[:n], idx_ref[:n])
        assert n == ref[0]["n_out"] and np.array_equal(idx[:n].cpu().numpy(), ref[0]["idx"])
        if r == 0:  # only [lo, hi) written so far
            for q in range(world):
                assert torch.isnan(bufs[q][:, hi:].float()).all()
                assert torch.equal(_bits(bufs[q][:, lo:hi]), _bits(Y_ref[:, lo:hi]))
    for q in range(world):
        assert torch.equal(_bits(bufs[q]), _bits(Y_ref)), f"buffer {q} differs"
        _check_oracle(bufs[q], ref)


def test_sharded_argument_checks():
    X, CB, SCB, b = _layer(8, 256, 64, 0, torch.float16, seed=1)
    Y = torch.empty((8, 128), dtype=torch.float16, device="cuda")
    ok = dict(path=native.PATH_AUTO)
    for ldY, off, dst in [(128, 4, [Y]),        # offset not a multiple of 8
                          (128, 72, [Y]),       # block runs past the row
                          (60, 0, [Y]),         # row shorter than the shard
                          (128, 0, [Y] * 9)]:   # too many destinations
        with pytest.raises((native.Int8mpError, ValueError)):
            native.int8_linear_forward_sharded(X, CB, SCB, b, 6.0, dst, ldY, off, **ok)
    native.int8_linear_forward_sharded(X, CB, SCB, b, 6.0, [Y], 128, 64, **ok)
    torch.cuda.synchronize()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("mode", ["nccl", "peer"])
def test_world_one_process_group_matches_unsharded(mode):
    X, CB, SCB, b, ref = _layer(64, 1024, 512, 4, torch.float16, seed=3, with_oracle=True)
    Y_ref, _, _, _ = native.int8_linear_forward(X, CB, SCB, b, 6.0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        layer = sharded.NShardedLinear(CB, SCB, b, T_max=128, mode=mode)
        for _ in range(2):
            Y = layer.forward(X, 6.0)
            torch.cuda.synchronize()
            assert layer.check_status()[0] == 0
            assert torch.equal(_bits(Y), _bits(Y_ref))
            _check_oracle(Y, ref)
        del layer
    finally:
        dist.destroy_process_group()
