"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Integer stages (CB, SCB, outlier idx / n_out, row codes Xq, row scales sA,
the fp16 gathers Xo / Wo, int32 accumulators) must match bit for bit; the fp16
output Y must satisfy max|Y - Yref| <= 1e-3 * max|Yref| + 2e-3.  The oracle
always quantises the weight itself from W; nothing it consumes comes from the
CUDA path.  Full-size configs compare sampled rows / output columns, chosen to
touch every 128 x 256 output tile.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import llm_int8 as O
from int8_mixed_precision_column_b200 import build, native, workloads

pytestmark = pytest.mark.gpu

PATHS = {"auto": native.PATH_AUTO, "tc": native.PATH_TENSOR_CORE, "decode": native.PATH_DECODE,
         "tc1": native.PATH_TENSOR_CORE_1SM}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    native.lib()


def to_np(t):
    return t.detach().cpu().numpy()


def gpu_forward(p, path="auto", workspace_fill=None):
    X = p.X.cuda()
    W = p.W.cuda()
    bias = p.bias.cuda() if p.bias is not None else None
    CB, SCB = native.int8_quantize_weight(W)
    ws = native.new_workspace(p.T, p.K, p.N)
    if workspace_fill is not None:
        ws.fill_(workspace_fill)
    Y, idx, n_out, ws = native.int8_linear_forward(X, CB, SCB, bias, p.threshold, workspace=ws, path=PATHS[path])
    st, where = native.int8_check_status(ws)
    assert st == 0, f"device status {st} at {where:#x} ({native.int8_last_cuda_error()})"
    v = native.workspace_views(ws, p.T, p.K, p.N)
    n = int(n_out.item())
    npad = (n + 63) // 64 * 64
    return {"Y": Y, "CB": CB, "SCB": SCB, "idx": to_np(idx[:n]), "n_out": n, "npad": npad,
            "Xq": v["Xq"], "sA": v["sA"], "Xo": v["Xo"], "Wo": v["Wo"], "ws": ws}


def check_forward(p, g, rows=None, cols=None, check_wo=True):
    """Compare GPU results against the oracle on the given rows / output columns."""
    X = p.X.cpu().numpy()
    cols = np.arange(p.N) if cols is None else np.asarray(cols)
    rows_sel = np.arange(p.T) if rows is None else np.asarray(rows)
    W_sel = p.W[torch.as_tensor(cols, device=p.W.device)].cpu().numpy()
    b_sel = p.bias[torch.as_tensor(cols, device=p.bias.device)].cpu().numpy() if p.bias is not None else None
    CBo, SCBo = O.quantize_weight(W_sel)
    assert np.array_equal(to_np(g["CB"][torch.as_tensor(cols, device="cuda")]), CBo)
    assert np.array_equal(to_np(g["SCB"][torch.as_tensor(cols, device="cuda")]), SCBo)
    r = O.linear_forward(X, CBo, SCBo, b_sel, p.threshold, rows=rows)
    assert g["n_out"] == r["n_out"]
    assert np.array_equal(g["idx"], r["idx"])
    rt = torch.as_tensor(rows_sel, device="cuda")
    assert np.array_equal(to_np(g["sA"][rt]), r["sA"])
    assert np.array_equal(to_np(g["Xq"][rt]), r["Xq"])
    n, npad = g["n_out"], g["npad"]
    if n:
        Xo = to_np(g["Xo"][rt, :npad])
        assert np.array_equal(Xo[:, :n], r["Xo"]) and np.all(Xo[:, n:] == 0)
        if check_wo:
            Wo = to_np(g["Wo"][torch.as_tensor(cols, device="cuda"), :npad])
            assert np.array_equal(Wo[:, :n], r["Wo"]) and np.all(Wo[:, n:] == 0)
    Y = to_np(g["Y"][rt][:, torch.as_tensor(cols, device="cuda")]).astype(np.float64)
    err = np.abs(Y - r["Y"]).max(initial=0.0)
    tol = O.y_tolerance(r["Y"])
    assert err <= tol, f"max|Y-Yref| = {err:.3g} > {tol:.3g}"
    return r


# ---------------------------------------------------------------------------
# weight quantisation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(64, 64), (48, 80), (272, 208), (4096, 4096), (16, 14336)])
def test_quantize_weight_bit_exact(N, K):
    g = torch.Generator().manual_seed(N * 7 + K)
    W = (torch.randn(N, K, generator=g) * 0.02).half()
    W[0] = 0
    W[1] = 0
    W[1, K // 2] = -3.0
    CB, SCB = native.int8_quantize_weight(W.cuda())
    CBo, SCBo = O.quantize_weight(W.numpy())
    assert np.array_equal(to_np(CB), CBo)
    assert np.array_equal(to_np(SCB), SCBo)


def test_quantize_weight_rounding_fixture(golden):
    g = golden("rounding_cases.txt")
    row = np.array([float(s) for s in g["row"]] + [0.0] * 8, dtype=np.float16)
    W = torch.from_numpy(np.tile(row, (16, 1)))
    CB, SCB = native.int8_quantize_weight(W.cuda())
    want = [int(s) for s in g["codes"]] + [0] * 8
    assert to_np(CB)[0].tolist() == want and float(SCB[0]) == 127.0


# ---------------------------------------------------------------------------
# forward: small and ragged shapes, both product kernels
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", ["auto", "tc", "decode"])
def test_toy(path):
    p = workloads.toy(seed=0)
    g = gpu_forward(p, path)
    r = check_forward(p, g, check_wo=(path == "tc"))
    assert g["idx"].tolist() == [3, 17] == r["idx"].tolist()


RAGGED = [
    # T, K, N, planted, threshold
    (1, 64, 64, 1, 6.0),
    (3, 16, 16, 0, 6.0),
    (17, 16, 32, 1, 6.0),
    (200, 208, 272, 3, 6.0),
    (130, 1024, 528, 17, 6.0),
    (300, 336, 512, 65, 6.0),
    (129, 512, 256, 16, 6.0),
    (256, 4096, 256, 64, 6.0),
]


@pytest.mark.parametrize("path", ["tc", "tc1"])
@pytest.mark.parametrize("T,K,N,planted,thr", RAGGED)
def test_ragged_tensor_core(T, K, N, planted, thr, path):
    p = workloads.make_problem("ragged", T, K, N, n_planted=planted, bias_std=0.01, threshold=thr, seed=T + K + N)
    check_forward(p, gpu_forward(p, path))


@pytest.mark.parametrize("T,N", [(1100, 8208), (513, 38416)])
def test_pair_tiles_outnumber_pairs(T, N):
    """More 256 x 512 output tiles than SM pairs, so pairs take several in turn
    (TMEM and the per-tile barriers reused with the outlier product added in
    place), two outlier K-blocks, and a ragged last tile in both directions
    (T = 1100: 76 rows; T = 513: one row; N: 16 columns), whose output the TMA
    stores clip.  Sampled rows against the oracle, every column."""
    p = workloads.make_problem("multi", T, 336, N, n_planted=70, bias_std=0.01, seed=T + N)
    g = gpu_forward(p, "tc")
    assert g["n_out"] > 64
    check_forward(p, g, rows=list(range(0, T, 37)) + [T - 1])


@pytest.mark.parametrize("T,K,N,planted,path", [
    (300, 20480, 256, 9, "tc"),       # K > 16384, few rows: two-pass CTA-per-row quantisation
    (2048, 20480, 128, 9, "tc"),      # K > 16384, many rows: warp-per-row quantisation
    (40, 131072, 64, 33, "tc"),       # the largest K the library takes
    (16, 131072, 64, 33, "decode"),   # ... through the one-kernel decode prep
    (3, 131072, 48, 2, "auto"),
])
def test_long_rows_and_maximum_k(T, K, N, planted, path):
    p = workloads.make_problem("longk", T, K, N, n_planted=planted, bias_std=0.01, seed=T + K)
    check_forward(p, gpu_forward(p, path), check_wo=path != "decode" and not (path == "auto" and T <= 16))


@pytest.mark.parametrize("T", [1, 2, 5, 8, 9, 15, 16])
def test_decode_matches_oracle_and_tensor_core(T):
    p = workloads.make_problem("dec", T, 1216, 400 - 400 % 16, n_planted=5, bias_std=0.01, seed=T)
    gd = gpu_forward(p, "decode")
    check_forward(p, gd, check_wo=False)
    gt = gpu_forward(p, "tc")
    assert np.array_equal(gd["idx"], gt["idx"])
    assert torch.equal(gd["Xq"], gt["Xq"]) and torch.equal(gd["sA"], gt["sA"])


@pytest.mark.parametrize("n_planted", [1, 15, 16, 17, 63, 64, 65, 130])
def test_outlier_count_padding_boundaries(n_planted):
    p = workloads.make_problem("pad", 160, 1024, 272, n_planted=n_planted, bias_std=0.01, seed=n_planted)
    g = gpu_forward(p, "tc")
    assert g["n_out"] >= n_planted
    check_forward(p, g)


@pytest.mark.parametrize("path", ["tc", "decode"])
def test_threshold_zero_is_pure_int8(path):
    p = workloads.make_problem("t0", 16, 256, 96, n_planted=4, bias_std=0.01, threshold=0.0, seed=3)
    g = gpu_forward(p, path)
    assert g["n_out"] == 0
    check_forward(p, g, check_wo=False)


@pytest.mark.parametrize("path", ["tc", "decode"])
def test_threshold_small_flags_every_column(path):
    p = workloads.make_problem("t01", 16, 128, 96, bias_std=0.01, threshold=0.1, seed=4)
    X = p.X
    X[X.abs() <= 0.1] = 0.5
    g = gpu_forward(p, path)
    assert g["n_out"] == 128 and g["idx"].tolist() == list(range(128))
    assert torch.count_nonzero(g["Xq"]).item() == 0
    check_forward(p, g, check_wo=(path == "tc"))


def test_zero_rows_and_outlier_only_rows():
    p = workloads.make_problem("zeros", 40, 256, 64, n_planted=2, bias_std=0.01, seed=5)
    p.X[3] = 0
    p.X[7] = 0
    p.X[7, p.planted_cols[0]] = 25.0
    g = gpu_forward(p, "tc")
    assert float(g["sA"][3]) == 0.0 and float(g["sA"][7]) == 0.0
    check_forward(p, g)


def test_exact_threshold_value_not_flagged():
    p = workloads.make_problem("edge", 8, 64, 32, seed=6)
    p.X[:, 10] = 6.0
    p.X[2, 20] = -6.0
    p.X[5, 30] = 6.00390625
    p.X.clamp_(-5.9, 5.9)
    p.X[:, 10] = 6.0
    p.X[2, 20] = -6.0
    p.X[5, 30] = 6.00390625
    g = gpu_forward(p, "auto")
    assert g["idx"].tolist() == [30]
    check_forward(p, g, check_wo=False)


@pytest.mark.parametrize("T,K,N,path,expect", [
    (1, 14336, 57344, "auto", "decode"), (16, 4096, 4096, "auto", "decode"),
    (17, 4096, 4096, "auto", "tc"), (2048, 4096, 4096, "auto", "tc"), (8192, 14336, 57344, "auto", "tc"),
    (4, 4096, 4096, "tc", "tc"), (2048, 4096, 4096, "tc1", "tc1"), (16, 4096, 4096, "decode", "decode"),
])
def test_product_kernel_choice(T, K, N, path, expect):
    """The automatic path: the decode GEMV for T <= 16, the SM-pair GEMM above
    (2-CTA clusters launch on B200); explicit paths are honoured."""
    assert native.int8_linear_product_kernel(T, K, N, PATHS[path]) == PATHS[expect]


def test_product_kernel_choice_rejects_bad_arguments():
    assert native.int8_linear_product_kernel(17, 4096, 4096, native.PATH_DECODE) == -1
    assert native.int8_linear_product_kernel(4, 4100, 4096, native.PATH_AUTO) == -1


def test_empty_batch():
    p = workloads.make_problem("empty", 0, 64, 64, seed=7)
    CB, SCB = native.int8_quantize_weight(p.W.cuda())
    Y, idx, n_out, ws = native.int8_linear_forward(p.X.cuda(), CB, SCB, None, 6.0)
    assert Y.shape == (0, 64) and int(n_out.item()) == 0


def test_workspace_contents_need_no_initialisation():
    p = workloads.make_problem("ws", 96, 512, 256, n_planted=5, bias_std=0.01, seed=8)
    a = gpu_forward(p, "tc", workspace_fill=0xFF)
    b = gpu_forward(p, "tc", workspace_fill=0x00)
    assert torch.equal(a["Y"], b["Y"]) and np.array_equal(a["idx"], b["idx"])
    check_forward(p, a)


def test_deterministic_repeat():
    p = workloads.make_problem("det", 300, 1024, 512, n_planted=9, bias_std=0.01, seed=9)
    X, W, bias = p.X.cuda(), p.W.cuda(), p.bias.cuda()
    CB, SCB = native.int8_quantize_weight(W)
    ws = native.new_workspace(p.T, p.K, p.N)
    Y1, idx1, n1, _ = native.int8_linear_forward(X, CB, SCB, bias, 6.0, workspace=ws)
    Y1 = Y1.clone()
    idx1 = idx1.clone()
    Y2, idx2, n2, _ = native.int8_linear_forward(X, CB, SCB, bias, 6.0, workspace=ws)
    assert torch.equal(Y1, Y2) and int(n1) == int(n2)
    assert torch.equal(idx1[: int(n1)], idx2[: int(n2)])


# ---------------------------------------------------------------------------
# int32 accumulators alone
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,K,N,path", [(16, 64, 64, "tc"), (200, 208, 272, "tc"), (384, 1536, 768, "tc"),
                                        (16, 14336, 512, "tc"), (16, 64, 64, "tc1"), (200, 208, 272, "tc1"),
                                        (384, 1536, 768, "tc1"), (600, 4096, 1040, "tc"), (1, 64, 64, "decode"),
                                        (16, 1216, 400, "decode"), (7, 14336, 256, "decode")])
def test_gemm_i32_bit_exact(T, K, N, path):
    g = torch.Generator().manual_seed(T * 3 + K)
    Xq = torch.randint(-127, 128, (T, K), generator=g, dtype=torch.int8)
    CB = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    Xq[0] = 127
    CB[0] = 127
    CB[-1] = -127
    acc = native.int8_gemm_i32(Xq.cuda(), CB.cuda(), path=PATHS[path])
    assert np.array_equal(to_np(acc), O.int8_matmul(Xq.numpy(), CB.numpy()))


# ---------------------------------------------------------------------------
# the configs at full size
# ---------------------------------------------------------------------------

def tile_rows(T, per_tile=2, tile=128):
    rows = []
    for m0 in range(0, T, tile):
        last = min(T, m0 + tile) - 1
        rows += [m0, last] if per_tile == 2 else list(np.linspace(m0, last, per_tile).astype(int))
    return np.unique(np.array(rows))


def tile_cols(N, per_tile=8, tile=256):
    cols = []
    for n0 in range(0, N, tile):
        last = min(N, n0 + tile) - 1
        cols += list(np.linspace(n0, last, per_tile).astype(int))
    return np.unique(np.array(cols))


@pytest.mark.parametrize("path", ["auto", "tc1"])
def test_llama7b_prefill_full(path):
    p = workloads.llama7b_prefill(seed=0)
    g = gpu_forward(p, path)
    r = check_forward(p, g)
    assert g["n_out"] == len(p.planted_cols) and r["idx"].tolist() == p.planted_cols
    acc = native.int8_gemm_i32(g["Xq"], g["CB"], path=PATHS["tc" if path == "auto" else path])
    assert np.array_equal(to_np(acc), r["acc"])


@pytest.mark.parametrize("n_dims,thr", [(0, 6.0), (8, 6.0), (64, 6.0), (512, 6.0), (8, 0.0), (8, 0.1)])
def test_density_sweep(n_dims, thr):
    p = workloads.density_sweep(n_dims, threshold=thr, seed=0, device="cuda")
    g = gpu_forward(p, "auto")
    rows = tile_rows(p.T, per_tile=2)
    check_forward(p, g, rows=rows, cols=tile_cols(p.N, per_tile=16))
    if thr == 0.1:
        assert g["n_out"] == p.K
    if thr == 0.0:
        assert g["n_out"] == 0


@pytest.mark.parametrize("T", [1, 4, 16])
def test_bloom_ffn_up_decode(T):
    p = workloads.bloom_ffn_up_decode(T, seed=0, device="cuda")
    g = gpu_forward(p, "auto")
    cols = tile_cols(p.N, per_tile=16)
    check_forward(p, g, cols=cols, check_wo=False)
    gt = gpu_forward(p, "tc")
    assert np.array_equal(g["idx"], gt["idx"])
    d = (g["Y"].float() - gt["Y"].float()).abs().max().item()
    assert d <= 1e-3 * gt["Y"].float().abs().max().item() + 2e-3


def test_bloom_ffn_up_prefill_sampled():
    """The headline config at full size (T=8192, K=14336, N=57344): every stage
    on sampled rows and columns that touch every output tile; then the int32
    accumulators of the pair kernel over the whole [8192, 57344] output (the
    same 256 x 512 tiles, persistent grid and raster as the forward, int32
    epilogue), bit for bit against the oracle's exact int8 product on 2 rows of
    every 128-row block and all 57344 columns, and CB bit for bit on every
    row of W."""
    p = workloads.bloom_ffn_up_prefill(8192, seed=0, device="cuda")
    g = gpu_forward(p, "auto")
    rows = tile_rows(p.T, per_tile=2)
    r = check_forward(p, g, rows=rows, cols=tile_cols(p.N, per_tile=8))
    acc = native.int8_gemm_i32(g["Xq"], g["CB"], path=PATHS["tc"])
    acc_rows = to_np(acc[torch.as_tensor(rows, device="cuda")])
    del acc
    chunk = 4096
    for j0 in range(0, p.N, chunk):
        CBo, _ = O.quantize_weight(p.W[j0: j0 + chunk].cpu().numpy())
        assert np.array_equal(to_np(g["CB"][j0: j0 + chunk]), CBo), j0
        assert np.array_equal(acc_rows[:, j0: j0 + chunk], O.int8_matmul(r["Xq"], CBo)), j0


def test_host_buffer_forward_matches_device_forward():
    p = workloads.llama7b_prefill(seed=1)
    g = gpu_forward(p, "auto")
    Xh = p.X.clone().pin_memory()
    Yh = torch.empty((p.T, p.N), dtype=torch.float16).pin_memory()
    idx_h = torch.empty((p.K,), dtype=torch.int32)
    n_h = torch.empty((1,), dtype=torch.int32)
    ws = torch.empty(native.int8_linear_forward_host_workspace_bytes(p.T, p.K, p.N), dtype=torch.uint8,
                     device="cuda")
    native.int8_linear_forward_host(Xh, g["CB"], g["SCB"], p.bias.cuda(), p.threshold, Yh, ws, idx_h, n_h)
    assert int(n_h) == g["n_out"]
    assert np.array_equal(idx_h.numpy()[: g["n_out"]], g["idx"])
    assert torch.equal(Yh, g["Y"].cpu())


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_async_host_forward_on_two_streams(dtype):
    """Non-blocking host-buffer forwards alternating on two streams and two
    workspaces (the pipelined e2e form) give the device forward's outputs."""
    p = workloads.llama7b_prefill(seed=2)
    X = p.X.to(dtype)
    W = p.W.to(dtype).cuda()
    b = p.bias.to(dtype).cuda()
    CB, SCB = native.int8_quantize_weight(W)
    Y_ref, idx_ref, n_ref, _ = native.int8_linear_forward(X.cuda(), CB, SCB, b, p.threshold)
    n = int(n_ref.item())
    Xh = X.clone().pin_memory()
    nbytes = native.int8_linear_forward_host_workspace_bytes(p.T, p.K, p.N)
    slots = [(torch.cuda.Stream(), torch.empty(nbytes, dtype=torch.uint8, device="cuda"),
              torch.empty((p.T, p.N), dtype=dtype).pin_memory(), torch.empty((p.K,), dtype=torch.int32).pin_memory(),
              torch.empty((1,), dtype=torch.int32).pin_memory()) for _ in range(2)]
    for i in range(5):
        s, ws, Yh, idx_h, n_h = slots[i % 2]
        native.int8_linear_forward_host_async(Xh, CB, SCB, b, p.threshold, Yh, ws, idx_h, n_h, stream=s)
    torch.cuda.synchronize()
    for s, ws, Yh, idx_h, n_h in slots:
        assert native.int8_check_status(ws)[0] == 0
        assert int(n_h) == n and torch.equal(idx_h[:n], idx_ref[:n].cpu())
        assert torch.equal(Yh.view(torch.int16), Y_ref.cpu().view(torch.int16))


def test_async_host_forward_rejects_pageable_buffers():
    p = workloads.toy(seed=0)
    CB, SCB = native.int8_quantize_weight(p.W.cuda())
    ws = torch.empty(native.int8_linear_forward_host_workspace_bytes(p.T, p.K, p.N), dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(ValueError):
        native.int8_linear_forward_host_async(p.X, CB, SCB, None, 6.0, torch.empty((p.T, p.N), dtype=torch.float16),
                                              ws)


# ---------------------------------------------------------------------------
# rounding and subnormal edge cases of the row codes and the outlier test
# ---------------------------------------------------------------------------

def _boundary_rows(seed=0, rows=48, K=512):
    """Rows whose products x * fp32(127/absmax) land on, just below and just
    above every k + 0.5 boundary, for a spread of absmax values."""
    rng = np.random.default_rng(seed)
    X = np.zeros((rows, K), np.float16)
    for r in range(rows):
        a = np.float16(127.0) if r == 0 else np.float16(rng.uniform(0.01, 100.0))
        inv = np.float32(127.0) / np.float32(a)
        vals = [a, -a]
        for k in range(0, 127):
            tgt = np.float16((k + 0.5) / float(inv))
            for v in (tgt, np.nextafter(tgt, np.float16(0)), np.nextafter(tgt, np.float16(np.inf))):
                if abs(float(v)) <= float(a):
                    vals += [v, -v]
        vals = np.array(vals[:K], np.float16)
        X[r, : vals.size] = vals
    return X


@pytest.mark.parametrize("path", ["tc", "decode"])
def test_row_codes_at_rounding_boundaries(path):
    X = _boundary_rows(rows=48 if path == "tc" else 16)
    T, K = X.shape
    W = (np.random.default_rng(1).normal(0, 0.02, (64, K))).astype(np.float16)
    p = workloads.LinearProblem("bounds", torch.from_numpy(X), torch.from_numpy(W), None, 1000.0)
    g = gpu_forward(p, path)
    mask = O.outlier_mask(X, 1000.0)
    Xq, sA = O.quantize_rows(X, mask)
    assert g["n_out"] == 0
    assert np.array_equal(to_np(g["sA"]), sA)
    assert np.array_equal(to_np(g["Xq"]), Xq)


@pytest.mark.parametrize("thr", [1e-6, 3e-5, 6.0])
def test_subnormal_rows_and_thresholds(thr):
    rng = np.random.default_rng(2)
    T, K, N = 24, 256, 64
    X = (rng.normal(0, 1, (T, K)) * 1e-6).astype(np.float16)   # mostly fp16 subnormals
    X[3] = (rng.normal(0, 1, K) * 2e-7).astype(np.float16)
    X[5, 7] = np.float16(6e-5)
    X[9] = 0
    X[9, 11] = np.float16(5.96e-8)                               # smallest subnormal
    W = rng.normal(0, 0.02, (N, K)).astype(np.float16)
    p = workloads.LinearProblem("subnormal", torch.from_numpy(X), torch.from_numpy(W), None, thr)
    for path in ("tc", "decode" if T <= 16 else "tc1"):
        check_forward(p, gpu_forward(p, path))
