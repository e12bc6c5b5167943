"""The row quantisation's rounding, restated on the CPU.

The kernels form a code as trunc(copysign(RZ(|y| + 0.5), y)), where RZ is the
fp32 addition rounded toward zero and y = x * fp32(127 / absmax) is the
round-to-nearest product (|y| <= 127.5).  With n = floor(|y| + 0.5), an integer
and so exact in fp32, the RZ sum lies in [n, n + 1), so this is round half away
from zero, the rounding the oracle takes for the absmax codes (Hugging Face
LLM.int8() integration page, section "Quantization mechanics": the scaled
value is rounded).  Here the RZ addition is emulated exactly (the fp64
sum of an fp32 and 0.5 is exact) and compared with the oracle's rounding.
"""
from __future__ import annotations

import numpy as np

from oracle import llm_int8 as O


def _rz_add_half(a: np.ndarray) -> np.ndarray:
    s = a.astype(np.float64) + 0.5            # exact: a is fp32 with |a| <= 127.5
    f = s.astype(np.float32)                  # nearest
    over = f.astype(np.float64) > s
    f[over] = np.nextafter(f[over], np.float32(0.0))   # largest fp32 <= s
    return f


def _kernel_code(y: np.ndarray) -> np.ndarray:
    return np.trunc(np.copysign(_rz_add_half(np.abs(y)), y)).astype(np.int64)


def _boundary_values() -> np.ndarray:
    k = np.arange(-128, 128, dtype=np.float32) + np.float32(0.5)
    out = [k]
    for direction in (np.inf, -np.inf):
        v = k
        for _ in range(4):
            v = np.nextafter(v, np.float32(direction))
            out.append(v)
    below_half = np.float32(0.5) - np.float32(2.0 ** -25) * np.arange(64, dtype=np.float32)
    out += [below_half, -below_half,
            np.array([0.0, -0.0, 2.0 ** -149, -(2.0 ** -149), 127.0, -127.0, 127.5, -127.5], np.float32)]
    y = np.concatenate(out).astype(np.float32)
    return y[np.abs(y) <= 127.5]


def test_rz_rounding_matches_round_half_away_at_boundaries():
    y = _boundary_values()
    assert np.array_equal(_kernel_code(y), O.round_half_away(y).astype(np.int64))


def test_rz_rounding_matches_round_half_away_random():
    y = np.random.default_rng(0).uniform(-127.5, 127.5, 1_000_000).astype(np.float32)
    assert np.array_equal(_kernel_code(y), O.round_half_away(y).astype(np.int64))


def test_nearest_addition_would_fail_below_one_half():
    # why the RZ addition: the round-to-nearest sum 0.49999997 + 0.5 is 1.0
    y = np.float32(0.5) - np.float32(2.0 ** -25)
    assert np.float32(y + np.float32(0.5)) == np.float32(1.0)
    assert _kernel_code(np.array([y], np.float32))[0] == 0 == O.round_half_away(np.array([y], np.float32))[0]
