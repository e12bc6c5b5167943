"""The plain C++ oracle (oracle/llm_int8_ref.cpp through oracle/cpp.py).

* Every pin of test_oracle_pins.py runs on it unchanged (the pins call the
  module-global ``O``, which these tests point at the C++ oracle).
* Its 16-bit conversions, written from the formats' definitions, are checked
  against numpy's own fp16 rounding for every fp16 pattern, every midpoint
  between neighbours and random values (numpy's float32 -> float16 cast rounds
  to nearest, ties to even), and against the bf16 rule pinned for the numpy
  oracle.
* On seeded problems it agrees with the numpy oracle: every integer stage and
  the 16-bit gathers bit for bit, Y within 1e-12 (both are fp64; only the
  summation order of the outlier dot products differs).
* Each planted mistake -- a textual edit of a copy of the C++ source, built
  into a temporary directory on the CPU -- is caught by at least one pin.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import test_oracle_pins as P
from oracle import cpp as C
from oracle import llm_int8 as N
from int8_mixed_precision_column_b200 import workloads


@pytest.fixture(scope="module")
def cpp():
    C.build()
    return C.Oracle(threads=4)


def check_fp16_conversions(o: C.Oracle):
    pats = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float32)
    got = o.to_f32(pats, C.F16)
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin]) and np.all(np.isnan(got[~fin]))
    # every finite fp16 value narrows back to its own pattern
    assert np.array_equal(o.from_f32(ref[fin], C.F16), pats[fin])
    # midpoints between neighbouring non-negative finite values (exact in fp32) and beyond
    pos = np.arange(0x7C00, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    rng = np.random.default_rng(0)
    rnd = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-5, 20000), rng.uniform(-70000, 70000, 5000),
                          [65504.0, 65519.0, 65520.0, 65536.0, 1e6, -65520.0, 2.0**-25, 3 * 2.0**-26]])
    x = np.concatenate([mids, -mids, rnd.astype(np.float32)])
    assert np.array_equal(o.from_f32(x, C.F16), x.astype(np.float16).view(np.uint16))


def check_bf16_conversions_match_numpy_oracle(o: C.Oracle):
    pats = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    a, b = o.to_f32(pats, C.BF16), N.bf16_to_f32(pats)
    fin = ~np.isnan(b)
    assert np.array_equal(a[fin], b[fin]) and np.all(np.isnan(a[~fin]))
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.normal(0, 10, 20000), rng.normal(0, 1e-38, 2000), [3.4e38, -3.39e38]]).astype(np.float32)
    assert np.array_equal(o.from_f32(x, C.BF16), N.f32_to_bf16(x))


def test_builds_and_loads(cpp):
    assert cpp.lib.oref_version() == 1 and cpp.Q_MAX == 127


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pins_hold_for_the_cpp_oracle(pin, golden, cpp, monkeypatch):
    monkeypatch.setattr(P, "O", cpp)
    P.run_pin(pin, golden)


def test_fp16_conversions(cpp):
    check_fp16_conversions(cpp)


def test_bf16_conversions(cpp):
    check_bf16_conversions_match_numpy_oracle(cpp)


# ---------------------------------------------------------------------------
# agreement with the numpy oracle
# ---------------------------------------------------------------------------

def _same(a: dict, b: dict, keys=("mask", "idx", "Xq", "sA", "Xo", "Wo", "acc")):
    assert a["n_out"] == b["n_out"]
    for k in keys:
        x, y = np.ascontiguousarray(a[k]), np.ascontiguousarray(b[k])
        assert x.dtype == y.dtype and x.shape == y.shape and np.array_equal(x.view(np.uint8), y.view(np.uint8)), k
    np.testing.assert_allclose(a["Y"], b["Y"], rtol=1e-12, atol=1e-13)


PROBLEMS = [
    # T, K, N, planted, lo, hi, threshold, bias, seed
    (16, 64, 64, 2, 8.0, 20.0, 6.0, True, 0),
    (37, 96, 40, 5, 6.0, 60.0, 6.0, True, 1),
    (9, 128, 48, 3, 6.0, 60.0, 0.0, False, 2),
    (7, 80, 32, 0, 6.0, 60.0, 0.1, True, 3),
    (50, 160, 96, 12, 6.0, 40.0, 6.0, True, 4),
]


@pytest.mark.parametrize("T,K,Nf,planted,lo,hi,thr,with_bias,seed", PROBLEMS)
def test_cpp_and_numpy_oracles_agree(cpp, T, K, Nf, planted, lo, hi, thr, with_bias, seed):
    p = workloads.make_problem("agree", T, K, Nf, n_planted=planted, lo=lo, hi=hi, bias_std=0.01 if with_bias else None,
                               threshold=thr, seed=seed)
    X, W = p.X.numpy(), p.W.numpy()
    X[1, 3] = 0.0
    X[2] = 0.0                                   # a zero row
    b = None if p.bias is None else p.bias.numpy()
    CBn, SCBn = N.quantize_weight(W)
    CBc, SCBc = cpp.quantize_weight(W)
    assert np.array_equal(CBn, CBc) and np.array_equal(SCBn, SCBc)
    _same(N.linear_forward(X, CBn, SCBn, b, thr), cpp.linear_forward(X, CBc, SCBc, b, thr))
    rows = [0, T - 1, T // 2]
    _same(N.linear_forward(X, CBn, SCBn, b, thr, rows=rows), cpp.linear_forward(X, CBc, SCBc, b, thr, rows=rows))
    _same(N.linear_forward_fp16w(X, W, b, thr), cpp.linear_forward_fp16w(X, W, b, thr))
    # bf16: the same values rounded to bf16 patterns
    Xb, Wb = N.f32_to_bf16(X.astype(np.float32)), N.f32_to_bf16(W.astype(np.float32))
    bb = None if b is None else N.f32_to_bf16(b.astype(np.float32))
    CBbn, SCBbn = N.quantize_weight_bf16(Wb)
    CBbc, SCBbc = cpp.quantize_weight_bf16(Wb)
    assert np.array_equal(CBbn, CBbc) and np.array_equal(SCBbn, SCBbc)
    _same(N.linear_forward_bf16(Xb, CBbn, SCBbn, bb, thr), cpp.linear_forward_bf16(Xb, CBbc, SCBbc, bb, thr))
    _same(N.linear_forward_fp16w_bf16(Xb, Wb, bb, thr), cpp.linear_forward_fp16w_bf16(Xb, Wb, bb, thr))


def test_int8_matmul_large_k_exact(cpp):
    K = 131072
    A = np.full((2, K), 127, np.int8)
    B = np.full((2, K), -127, np.int8)
    B[1] = 127
    acc = cpp.int8_matmul(A, B)
    assert acc[0, 0] == -K * 16129 and acc[0, 1] == K * 16129
    g = torch.Generator().manual_seed(3)
    A = torch.randint(-127, 128, (5, 333), generator=g, dtype=torch.int8).numpy()
    B = torch.randint(-127, 128, (7, 333), generator=g, dtype=torch.int8).numpy()
    assert np.array_equal(cpp.int8_matmul(A, B), N.int8_matmul(A, B))


# ---------------------------------------------------------------------------
# planted mistakes: a copy of the C++ source with one edit, built on the CPU
# ---------------------------------------------------------------------------

CPP_PLANTS = {
    "round_half_even": ("float q = std::round(y);", "float q = std::nearbyint(y);"),
    "threshold_ge": ("> threshold) mask[k] = 1;", ">= threshold) mask[k] = 1;"),
    "absmax_over_all_columns": ("      if (!mask[k]) am = std::fmax(am,", "      am = std::fmax(am,"),
    "dequant_by_127_once": ("y = y / 16129.0;", "y = y / 127.0;"),
    "outlier_term_dropped": ("y = y + o;", "y = y + 0.0 * o;"),
    "outlier_sign_flipped": ("y = y + o;", "y = y - o;"),
    "weight_row_reversed": ("static_cast<int64_t>(CB[j * K + k])", "static_cast<int64_t>(CB[j * K + (K - 1 - k)])"),
    "outlier_weight_misindexed": ("CB[j * K + idx[o]]", "CB[j * K + idx[(o + 1) % n_out]]"),
    "fp16_ties_away": ("(r == 0.5 && std::fmod(n, 2.0) != 0.0)", "(r == 0.5)"),
    "fp16_subnormal_scale": ("std::ldexp(static_cast<float>(m), -24)", "std::ldexp(static_cast<float>(m), -25)"),
}


@pytest.mark.parametrize("plant", sorted(CPP_PLANTS))
def test_planted_mistake_in_cpp_oracle_is_caught(plant, golden, monkeypatch, tmp_path):
    old, new = CPP_PLANTS[plant]
    src = open(C.SRC).read()
    assert src.count(old) == 1, plant
    path = tmp_path / "llm_int8_ref_planted.cpp"
    path.write_text(src.replace(old, new))
    bad = C.Oracle(C.compile_source(str(path), str(tmp_path / "lib" / "liboracle_planted.so")), threads=2)
    monkeypatch.setattr(P, "O", bad)
    caught = []
    checks = [lambda g, pin=pin: P.run_pin(pin, g) for pin in P.ALL_PINS]
    checks += [lambda g: check_fp16_conversions(bad), lambda g: check_bf16_conversions_match_numpy_oracle(bad)]
    for i, chk in enumerate(checks):
        try:
            chk(golden)
        except (AssertionError, ValueError, IndexError, OverflowError):
            caught.append(i)
    assert caught, f"no pin caught the planted mistake {plant}"
