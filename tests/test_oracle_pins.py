"""Pins for the CPU oracle against what the pages and the mathematics fix.

Each ``check_*`` function is a pin; the ``test_*`` functions run them on the
oracle as written, and ``test_planted_*`` runs them on an oracle with a
deliberately planted mistake (on the CPU) to show the pin catches it.
"""

from __future__ import annotations

import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import llm_int8 as O
from int8_mixed_precision_column_b200 import workloads


def f16(a):
    return np.asarray(a, dtype=np.float16)


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def check_worked_example(read_golden):
    """Absmax worked example (HF integration page, "Quantization mechanics")."""
    g = read_golden("absmax_worked_example.txt")
    v = f16([float(s) for s in g["vector"]])
    CB, SCB = O.quantize_weight(v[None, :])
    scale = 127.0 / float(SCB[0])
    assert abs(scale - float(g["scale_printed"][0])) <= float(g["scale_printed_tolerance"][0])
    lo, hi = (int(s) for s in g["code_range"])
    assert CB.min() >= lo and CB.max() <= hi
    assert CB[0].tolist() == [int(s) for s in g["codes_derived"]]
    # the same rule applied row-wise to activations, with no outliers
    Xq, sA = O.quantize_rows(v[None, :], np.zeros(v.size, bool))
    assert Xq[0].tolist() == [int(s) for s in g["codes_derived"]]
    assert sA[0] == SCB[0]


def check_rounding(read_golden):
    """Ties round away from zero; absmax 127 makes the multiplier exactly 1."""
    g = read_golden("rounding_cases.txt")
    row = f16([float(s) for s in g["row"]])
    want = [int(s) for s in g["codes"]]
    CB, SCB = O.quantize_weight(row[None, :])
    assert SCB[0] == 127.0
    assert CB[0].tolist() == want
    Xq, sA = O.quantize_rows(row[None, :], np.zeros(row.size, bool))
    assert Xq[0].tolist() == want


def check_range_and_absmax():
    rng = np.random.default_rng(1)
    W = f16(rng.normal(0, 1, (33, 71)))
    CB, SCB = O.quantize_weight(W)
    assert np.abs(CB.astype(int)).max() <= 127
    j = np.arange(W.shape[0])
    k = np.abs(W.astype(np.float32)).argmax(axis=1)
    assert np.all(np.abs(CB[j, k].astype(int)) == 127)
    assert np.all(np.sign(CB[j, k]) == np.sign(W[j, k]))
    assert np.array_equal(SCB, np.abs(W.astype(np.float32)).max(axis=1))


def check_recovery_half_step():
    """|W - CB*SCB/127| <= SCB/254: recovery to within half a quantisation step."""
    rng = np.random.default_rng(2)
    W = f16(rng.normal(0, 0.02, (40, 96)))
    W[3] = 0  # zero row: scale 0, all codes 0, exact recovery
    CB, SCB = O.quantize_weight(W)
    rec = CB.astype(np.float64) * SCB.astype(np.float64)[:, None] / 127.0
    err = np.abs(W.astype(np.float64) - rec)
    bound = SCB.astype(np.float64)[:, None] / 254.0 * (1 + 1e-6)
    assert np.all(err <= bound)
    assert np.all(CB[3] == 0) and SCB[3] == 0


def bruteforce_mask(X, thr):
    T, K = X.shape
    out = []
    for k in range(K):
        hit = False
        for t in range(T):
            if thr > 0 and abs(float(X[t, k])) > thr:
                hit = True
        out.append(hit)
    return np.array(out, dtype=bool)


def check_mask_bruteforce():
    rng = np.random.default_rng(3)
    X = f16(rng.normal(0, 3, (7, 13)))
    X[2, 5] = 6.0   # exactly the threshold: "exceeds" is strict, not flagged
    X[4, 5] = -6.0
    X[0, 9] = np.float16(6.00390625)  # next fp16 above 6: flagged
    X[:, 11] = 0.0
    for thr in (6.0, 2.5, 0.1, 0.0, -1.0):
        m = O.outlier_mask(X, thr)
        assert np.array_equal(m, bruteforce_mask(X, thr)), thr
    m6 = O.outlier_mask(X, 6.0)
    assert m6[9] and not (m6[5] and np.abs(X[:, 5].astype(np.float32)).max() <= 6.0)
    assert O.outlier_index(m6).tolist() == sorted(np.nonzero(m6)[0].tolist())


def check_toy_columns():
    p = workloads.toy(seed=0)
    idx = O.outlier_index(O.outlier_mask(p.X.numpy(), p.threshold))
    assert idx.tolist() == [3, 17]


def check_issue_1609(read_golden):
    """threshold 0.1 flags every column of a randn(2, 8) activation."""
    g = read_golden("issue1609_threshold.txt")
    k, n, t = int(g["in_features"][0]), int(g["out_features"][0]), int(g["tokens"][0])
    thr = float(g["threshold"][0])
    gen = torch.Generator().manual_seed(42)
    x = torch.randn(t, k, generator=gen).half().numpy()
    W = torch.randn(n, k, generator=gen).half().numpy() * np.float16(0.3)
    CB, SCB = O.quantize_weight(W)
    r = O.linear_forward(x, CB, SCB, None, thr)
    assert r["idx"].tolist() == [int(s) for s in g["idx_printed"]]
    assert np.all(r["Xq"] == 0)


def check_threshold_off():
    rng = np.random.default_rng(4)
    X = f16(rng.normal(0, 10, (5, 16)))
    for thr in (0.0, -3.0, float("nan")):
        assert O.outlier_mask(X, thr).sum() == 0


def check_idx_ignores_weights():
    """The threshold acts on activations only (issue #1609 answer)."""
    p = workloads.toy(seed=5)
    X, W = p.X.numpy(), p.W.numpy()
    r1 = O.linear_forward(X, *O.quantize_weight(W), None, 6.0)
    W2 = (W[::-1, ::-1] * np.float16(50.0)).astype(np.float16)
    r2 = O.linear_forward(X, *O.quantize_weight(W2), None, 6.0)
    assert np.array_equal(r1["idx"], r2["idx"])
    assert np.array_equal(r1["Xq"], r2["Xq"]) and np.array_equal(r1["sA"], r2["sA"])


def exact_code(x: float, absmax: float) -> int:
    """Nearest integer to x*127/absmax in exact rationals, ties away from zero."""
    if absmax == 0:
        return 0
    v = Fraction(x) * 127 / Fraction(absmax)
    a = abs(v)
    q = int(a)
    if a - q >= Fraction(1, 2):
        q += 1
    q = min(q, 127)
    return q if v >= 0 else -q


def check_rowquant_bruteforce():
    """Row absmax over non-outlier columns, outlier columns coded 0 (loops)."""
    rng = np.random.default_rng(6)
    X = f16(rng.normal(0, 1, (9, 23)))
    X[:, 4] = f16(rng.uniform(7, 30, 9))
    X[3, 17] = -9.0
    X[6, :] = 0.0
    X[8, :] = 0.0
    X[8, 4] = 11.0  # only an outlier in this row: absmax of the rest is 0
    mask = O.outlier_mask(X, 6.0)
    Xq, sA = O.quantize_rows(X, mask)
    T, K = X.shape
    for t in range(T):
        am = 0.0
        for k in range(K):
            if not mask[k]:
                am = max(am, abs(float(X[t, k])))
        assert float(sA[t]) == am
        for k in range(K):
            want = 0 if mask[k] else exact_code(float(X[t, k]), am)
            assert int(Xq[t, k]) == want, (t, k)


def check_int8_matmul_bruteforce():
    rng = np.random.default_rng(7)
    A = rng.integers(-127, 128, (5, 37)).astype(np.int8)
    B = rng.integers(-127, 128, (6, 37)).astype(np.int8)
    acc = O.int8_matmul(A, B)
    for t, j in itertools.product(range(5), range(6)):
        assert int(acc[t, j]) == sum(int(A[t, k]) * int(B[j, k]) for k in range(37))
    # extreme magnitude: K * 127^2 without overflow
    K = 14336
    A = np.full((2, K), 127, np.int8)
    B = np.full((3, K), -127, np.int8)
    B[1] = 127
    acc = O.int8_matmul(A, B)
    assert acc.dtype == np.int32
    assert acc[0, 0] == -K * 16129 and acc[1, 1] == K * 16129


def lossless_problem(seed, with_outliers):
    """Integer X, W whose quantisation is exact: every row has absmax 127."""
    rng = np.random.default_rng(seed)
    T, K, N = 6, 40, 9
    X = rng.integers(-127, 128, (T, K)).astype(np.float64)
    X[np.arange(T), rng.integers(0, K, T)] = 127.0 * rng.choice([-1, 1], T)
    W = rng.integers(-127, 128, (N, K)).astype(np.float64)
    W[np.arange(N), rng.integers(0, K, N)] = 127.0 * rng.choice([-1, 1], N)
    cols = []
    if with_outliers:
        cols = [2, 31]
        X[:, cols] = rng.choice([-1, 1], (T, 2)) * rng.integers(151, 400, (T, 2))
        for t in range(T):  # keep a 127 outside the outlier columns
            if np.abs(np.delete(X[t], cols)).max() < 127:
                X[t, 0] = 127.0
    b = rng.integers(-50, 50, N).astype(np.float64)
    return f16(X), f16(W), f16(b), cols


def check_lossless_closed_form():
    """When quantisation is lossless, Y is exactly X @ W^T + b."""
    for with_out in (False, True):
        X, W, b, cols = lossless_problem(11 + with_out, with_out)
        CB, SCB = O.quantize_weight(W)
        assert np.all(SCB == 127.0) and np.array_equal(CB.astype(np.float64), W.astype(np.float64))
        thr = 150.0 if with_out else 0.0
        r = O.linear_forward(X, CB, SCB, b, thr)
        assert r["idx"].tolist() == cols
        exact = X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)
        assert np.array_equal(r["Y"], exact)


def check_all_columns_flagged():
    """n_out = K: the int8 part vanishes and Y = X @ fp16(CB*SCB/127)^T + b."""
    p = workloads.make_problem("allcols", 12, 48, 20, w_std=0.05, bias_std=0.01, seed=9)
    X = p.X.numpy()
    X[np.abs(X) <= 0.1] = np.float16(0.5)
    CB, SCB = O.quantize_weight(p.W.numpy())
    r = O.linear_forward(X, CB, SCB, p.bias.numpy(), 0.1)
    assert r["n_out"] == 48 and np.all(r["Xq"] == 0) and np.all(r["acc"] == 0)
    Wdq = np.empty(CB.shape, np.float16)
    for j in range(CB.shape[0]):
        for k in range(CB.shape[1]):
            Wdq[j, k] = np.float16(np.float32(np.float32(CB[j, k]) * SCB[j]) / np.float32(127))
    want = X.astype(np.float64) @ Wdq.astype(np.float64).T + p.bias.numpy().astype(np.float64)
    np.testing.assert_allclose(r["Y"], want, rtol=1e-12, atol=1e-12)


def check_pure_int8_path():
    """threshold 0: Y equals the product of the dequantised int8 operands."""
    p = workloads.make_problem("pure", 10, 64, 24, n_planted=3, bias_std=0.01, seed=10)
    X = p.X.numpy()
    CB, SCB = O.quantize_weight(p.W.numpy())
    r = O.linear_forward(X, CB, SCB, p.bias.numpy(), 0.0)
    assert r["n_out"] == 0 and r["Xo"].shape[1] == 0
    Xd = r["Xq"].astype(np.float64) * r["sA"].astype(np.float64)[:, None] / 127.0
    Wd = CB.astype(np.float64) * SCB.astype(np.float64)[:, None] / 127.0
    want = Xd @ Wd.T + p.bias.numpy().astype(np.float64)
    np.testing.assert_allclose(r["Y"], want, rtol=1e-10, atol=1e-12)


def check_bias_linearity():
    p = workloads.toy(seed=3)
    X = p.X.numpy()
    CB, SCB = O.quantize_weight(p.W.numpy())
    y1 = O.linear_forward(X, CB, SCB, p.bias.numpy(), 6.0)["Y"]
    y0 = O.linear_forward(X, CB, SCB, None, 6.0)["Y"]
    np.testing.assert_allclose(y1 - y0, np.broadcast_to(p.bias.numpy().astype(np.float64), y1.shape),
                               rtol=0, atol=1e-12)


def check_error_bound():
    """|Y - (X W^T + b)| stays within the bound the quantisation steps imply."""
    p = workloads.make_problem("bound", 16, 256, 32, n_planted=4, lo=6.0, hi=40.0,
                               w_std=0.02, bias_std=0.01, seed=12)
    X, W, b = p.X.numpy(), p.W.numpy(), p.bias.numpy()
    CB, SCB = O.quantize_weight(W)
    r = O.linear_forward(X, CB, SCB, b, 6.0)
    exact = X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)
    ax = np.abs(X.astype(np.float64))
    aw = np.abs(W.astype(np.float64))
    m = r["mask"]
    ex = r["sA"].astype(np.float64)[:, None] / 254.0          # per-row activation step / 2
    ew = SCB.astype(np.float64)[:, None] / 254.0               # per-row weight step / 2
    nonout = (~m).astype(np.float64)
    bound = (ax * nonout) @ np.broadcast_to(ew, W.shape).T + (np.broadcast_to(ex, X.shape) * nonout) @ aw.T \
        + (np.broadcast_to(ex, X.shape) * nonout) @ np.broadcast_to(ew, W.shape).T
    outm = m.astype(np.float64)
    bound = bound + (ax * outm) @ (np.broadcast_to(ew, W.shape) + aw * 2.0**-10).T
    err = np.abs(r["Y"] - exact)
    assert np.all(err <= bound * (1 + 1e-5) + 1e-9)
    assert err.max() > 0  # quantisation is genuinely lossy here


def check_outlier_operands():
    p = workloads.toy(seed=0)
    X = p.X.numpy()
    CB, SCB = O.quantize_weight(p.W.numpy())
    r = O.linear_forward(X, CB, SCB, p.bias.numpy(), 6.0)
    assert r["Xo"].shape == (16, 2) and r["Wo"].shape == (64, 2)
    for oi, k in enumerate([3, 17]):
        assert np.array_equal(r["Xo"][:, oi], X[:, k])
        for j in range(64):
            v = np.float16(np.float32(np.float32(int(CB[j, k])) * SCB[j]) / np.float32(127))
            assert r["Wo"][j, oi] == v


def check_fp16w_all_columns_is_exact_product():
    """has_fp16_weights=True, every column flagged: Y = X @ W^T + b exactly."""
    p = workloads.make_problem("fp16w", 10, 48, 24, w_std=0.05, bias_std=0.01, seed=13)
    X = p.X.numpy()
    X[np.abs(X) <= 0.1] = np.float16(0.5)
    W, b = p.W.numpy(), p.bias.numpy()
    r = O.linear_forward_fp16w(X, W, b, 0.1)
    assert r["n_out"] == 48 and np.all(r["acc"] == 0)
    exact = X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)
    np.testing.assert_allclose(r["Y"], exact, rtol=1e-12, atol=1e-12)


def check_fp16w_without_outliers_equals_int8_forward():
    p = workloads.make_problem("fp16w0", 9, 64, 32, n_planted=3, bias_std=0.01, seed=14)
    X, W, b = p.X.numpy(), p.W.numpy(), p.bias.numpy()
    r = O.linear_forward_fp16w(X, W, b, 0.0)
    r8 = O.linear_forward(X, *O.quantize_weight(W), b, 0.0)
    assert np.array_equal(r["Y"], r8["Y"]) and r["n_out"] == 0


def check_fp16w_outlier_weights_are_the_fp16_columns():
    X, W, b, cols = lossless_problem(21, True)
    W = W.astype(np.float16)
    W[:, cols] = np.float16(0.3333)          # not representable as CB*SCB/127 with SCB = 127
    W[:, 0] = np.float16(127.0)              # keep each row's absmax (127) in a non-outlier column
    r = O.linear_forward_fp16w(X, W, b, 150.0)
    assert r["idx"].tolist() == cols and np.array_equal(r["Wo"], W[:, cols])
    exact = X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)
    np.testing.assert_allclose(r["Y"], exact, rtol=0, atol=1e-9)


def check_bf16_conversions():
    """Widening is exact; narrowing picks the nearest bf16, ties to the even pattern."""
    pats = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    f = O.bf16_to_f32(pats)
    ok = ~np.isnan(f)
    assert np.array_equal(O.f32_to_bf16(f[ok]), pats[ok])
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(0, 10, 20000), rng.normal(0, 1e-30, 2000)]).astype(np.float32)
    mid = (O.bf16_to_f32(pats[:0x7F80].astype(np.uint16)).astype(np.float64))  # non-negative finite
    b = O.f32_to_bf16(x)
    got = O.bf16_to_f32(b).astype(np.float64)
    ax = np.abs(x.astype(np.float64))
    lo_i = np.clip(np.searchsorted(mid, ax, side="right") - 1, 0, mid.size - 2)
    lo, hi = mid[lo_i], mid[lo_i + 1]
    best = np.where(ax - lo < hi - ax, lo, np.where(ax - lo > hi - ax, hi, np.where(lo_i % 2 == 0, lo, hi)))
    assert np.array_equal(np.abs(got), best)


def check_bf16_worked_example(read_golden):
    g = read_golden("absmax_worked_example.txt")
    v = O.f32_to_bf16(np.array([float(t) for t in g["vector"]], np.float32))
    CB, SCB = O.quantize_weight_bf16(v[None, :])
    assert abs(127.0 / float(SCB[0]) - float(g["scale_printed"][0])) <= float(g["scale_printed_tolerance"][0])
    assert CB[0].tolist() == [int(t) for t in g["codes_derived"]]


def check_bf16_lossless_closed_form():
    for with_out in (False, True):
        X, W, b, cols = lossless_problem(31 + with_out, with_out)   # integers: exact in bf16 too
        Xb, Wb, bb = (O.f32_to_bf16(a.astype(np.float32)) for a in (X, W, b))
        CB, SCB = O.quantize_weight_bf16(Wb)
        r = O.linear_forward_bf16(Xb, CB, SCB, bb, 150.0 if with_out else 0.0)
        assert r["idx"].tolist() == cols
        # outlier magnitudes up to 400 are not all bf16 integers: use the bf16 values
        Xv, Wv, bv = (O.bf16_to_f32(a).astype(np.float64) for a in (Xb, Wb, bb))
        exact = Xv @ Wv.T + bv
        assert np.array_equal(r["Y"], exact)


def check_bf16_all_columns_flagged():
    rng = np.random.default_rng(8)
    X = O.f32_to_bf16(rng.choice([-1.0, 1.0], (6, 32)).astype(np.float32) * rng.uniform(0.2, 3, (6, 32)).astype(np.float32))
    W = O.f32_to_bf16(rng.normal(0, 0.05, (16, 32)).astype(np.float32))
    CB, SCB = O.quantize_weight_bf16(W)
    r = O.linear_forward_bf16(X, CB, SCB, None, 0.1)
    assert r["n_out"] == 32 and np.all(r["acc"] == 0)
    Wdq = np.empty(CB.shape, np.float32)
    for j in range(CB.shape[0]):
        for k in range(CB.shape[1]):
            Wdq[j, k] = np.float32(np.float32(CB[j, k]) * SCB[j]) / np.float32(127)
    want = O.bf16_to_f32(X).astype(np.float64) @ O.bf16_to_f32(O.f32_to_bf16(Wdq)).astype(np.float64).T
    np.testing.assert_allclose(r["Y"], want, rtol=1e-12, atol=1e-12)


def check_bf16_fp16w_all_columns_is_exact_product():
    """bf16 has_fp16_weights=True with every column an outlier: Y = X W^T + bias
    over the bf16 values, exactly (the int8 part is all zero)."""
    rng = np.random.default_rng(9)
    X = O.f32_to_bf16(rng.choice([-1.0, 1.0], (5, 48)).astype(np.float32) * rng.uniform(0.5, 4, (5, 48)).astype(np.float32))
    W = O.f32_to_bf16(rng.normal(0, 0.05, (32, 48)).astype(np.float32))
    b = O.f32_to_bf16(rng.normal(0, 0.1, 32).astype(np.float32))
    r = O.linear_forward_fp16w_bf16(X, W, b, 0.25)
    assert r["n_out"] == 48 and np.all(r["acc"] == 0) and np.array_equal(r["Wo"], W)
    want = np.empty((5, 32))
    for t in range(5):
        for j in range(32):
            want[t, j] = sum(float(O.bf16_to_f32(X[t, k])) * float(O.bf16_to_f32(W[j, k])) for k in range(48))
            want[t, j] += float(O.bf16_to_f32(b[j]))
    np.testing.assert_allclose(r["Y"], want, rtol=1e-12, atol=1e-12)


def check_bf16_fp16w_without_outliers_is_int8_forward():
    """With the decomposition off, the bf16 weight only enters through CB/SCB."""
    rng = np.random.default_rng(10)
    X = O.f32_to_bf16(rng.normal(0, 1, (7, 64)).astype(np.float32))
    W = O.f32_to_bf16(rng.normal(0, 0.02, (48, 64)).astype(np.float32))
    r = O.linear_forward_fp16w_bf16(X, W, None, 0.0)
    CB, SCB = O.quantize_weight_bf16(W)
    q = O.linear_forward_bf16(X, CB, SCB, None, 0.0)
    assert r["n_out"] == 0 and np.array_equal(r["CB"], CB)
    np.testing.assert_array_equal(r["Y"], q["Y"])


ALL_PINS = [
    check_worked_example, check_rounding, check_range_and_absmax, check_recovery_half_step,
    check_mask_bruteforce, check_toy_columns, check_issue_1609, check_threshold_off,
    check_idx_ignores_weights, check_rowquant_bruteforce, check_int8_matmul_bruteforce,
    check_lossless_closed_form, check_all_columns_flagged, check_pure_int8_path,
    check_bias_linearity, check_error_bound, check_outlier_operands,
    check_fp16w_all_columns_is_exact_product, check_fp16w_without_outliers_equals_int8_forward,
    check_fp16w_outlier_weights_are_the_fp16_columns,
    check_bf16_conversions, check_bf16_worked_example, check_bf16_lossless_closed_form,
    check_bf16_all_columns_flagged, check_bf16_fp16w_all_columns_is_exact_product,
    check_bf16_fp16w_without_outliers_is_int8_forward,
]


def run_pin(pin, read_golden):
    if "read_golden" in pin.__code__.co_varnames[: pin.__code__.co_argcount]:
        pin(read_golden)
    else:
        pin()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, golden):
    run_pin(pin, golden)


def test_oracle_exports():
    assert oracle.Q_MAX == 127
    assert oracle.y_tolerance(np.array([[10.0, -20.0]])) == pytest.approx(0.022)


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin
# ---------------------------------------------------------------------------

_ORIG = {n: getattr(O, n) for n in ("combine", "outlier_operands", "absmax_codes")}


def _half_even(v):
    return np.round(np.asarray(v, dtype=np.float32).astype(np.float64))


def _mask_ge(X, threshold):
    thr = np.float32(threshold)
    if not thr > 0:
        return np.zeros(X.shape[1], bool)
    return (np.abs(np.asarray(X, np.float16).astype(np.float32)) >= thr).any(axis=0)


def _rows_all_cols(X, mask):
    Xf = np.asarray(X, np.float16).astype(np.float32)
    sA = np.abs(Xf).max(axis=1).astype(np.float32)
    Xq = _ORIG["absmax_codes"](np.where(mask[None, :], np.float32(0), Xf), sA)
    Xq[:, mask] = 0
    return Xq, sA


def _combine_one_127(acc, sA, SCB, Xo, Wo, bias):
    return _ORIG["combine"](acc, sA, SCB, Xo, Wo, bias) * 127.0


def _combine_no_outliers(acc, sA, SCB, Xo, Wo, bias):
    return _ORIG["combine"](acc, sA, SCB, Xo[:, :0], Wo[:, :0], bias)


def _combine_sign(acc, sA, SCB, Xo, Wo, bias):
    return _ORIG["combine"](acc, sA, SCB, Xo, -Wo, bias)


def _matmul_transposed(Xq, CB):
    return (Xq.astype(np.float64) @ CB.astype(np.float64)).astype(np.int64).astype(np.int32)


def _operands_shifted(X, CB, SCB, idx):
    Xo, Wo = _ORIG["outlier_operands"](X, CB, SCB, idx)
    return Xo, np.roll(Wo, 1, axis=1)


PLANTS = {
    "round_half_even": ("round_half_away", _half_even),
    "threshold_ge": ("outlier_mask", _mask_ge),
    "absmax_over_all_columns": ("quantize_rows", _rows_all_cols),
    "dequant_by_127_once": ("combine", _combine_one_127),
    "outlier_term_dropped": ("combine", _combine_no_outliers),
    "outlier_sign_flipped": ("combine", _combine_sign),
    "transposed_weight": ("int8_matmul", _matmul_transposed),
    "outlier_weight_misindexed": ("outlier_operands", _operands_shifted),
}


@pytest.mark.parametrize("plant", sorted(PLANTS))
def test_planted_mistake_is_caught(plant, golden, monkeypatch):
    name, fake = PLANTS[plant]
    monkeypatch.setattr(O, name, fake)
    caught = []
    for pin in ALL_PINS:
        try:
            run_pin(pin, golden)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {plant}"
