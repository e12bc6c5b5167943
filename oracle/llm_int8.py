"""CPU oracle for the LLM.int8() forward linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never calls it, and this module imports nothing from the
product package.

It restates, step by step and in plain numpy, what the pages describe:

* "Hugging Face integrates LLM.int8() ... into Transformers and Accelerate",
  section "Core idea of LLM.int8()": (1) outlier extraction per column of
  the hidden state, (2) int8 vector-wise matmul for the rest (row-wise for
  activations, column-wise for weights) and fp16 matmul for the outliers,
  (3) dequantise and sum into an fp16 result.
* same page, section "Quantization mechanics": absmax quantisation, scale
  127/absmax, codes in [-127, 127]; and the weight recovery
  ``CB * SCB / 127`` under "Integration into transformers".
* bitsandbytes ``Linear8bitLt`` docstring, ``threshold`` argument: activation
  columns where any value exceeds the threshold take the fp16 path.
* bitsandbytes issue #1609: ``state.idx`` lists the outlier columns of the
  last forward; the threshold acts on activations, not weights.
* inference-research record "LLM.int8() / bitsandbytes int8", Activation
  scheme: separate normalisation constants per inner product; outlier
  feature dimensions go to a second 16-bit matmul.

Readings taken where the pages are silent:
threshold <= 0 disables the decomposition; "exceeds" is strict ``>``;
a column is an outlier for every token if any token exceeds; the row absmax
runs over non-outlier columns only; rounding is half away from zero after an
fp32 multiply by the fp32 quotient 127/absmax; a zero absmax gives all-zero
codes; SCB holds the fp32 absmax; the outlier weights are fp16 rounded from
the fp32 value ``(CB * SCB) / 127``.

Every float that decides an integer code is computed in fp32 (the kernel's
precision); the reference output Y is computed in fp64.  The int8 product is
exact: it is evaluated as an fp64 matmul of small integers whose partial sums
stay below 2**53, so no rounding can occur.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
(worked example, rounding cases, closed forms, brute force).
"""

from __future__ import annotations

import numpy as np

Q_MAX = 127  # int8 codes live in [-127, 127] (symmetric, -128 unused)


# ---------------------------------------------------------------------------
# Scalar building blocks
# ---------------------------------------------------------------------------

def round_half_away(v: np.ndarray) -> np.ndarray:
    """Round to nearest, ties away from zero (C ``roundf``), returned as float64.

    The fp32 input is widened to fp64, where ``|v| + 0.5`` is exact for every
    fp32 value, so the floor gives the correctly rounded integer.
    """
    v64 = np.asarray(v, dtype=np.float32).astype(np.float64)
    return np.sign(v64) * np.floor(np.abs(v64) + 0.5)


def absmax_codes(values_f32: np.ndarray, absmax_f32: np.ndarray) -> np.ndarray:
    """Absmax quantisation of fp32 values given their fp32 absmax (per row).

    "Quantization mechanics" (absmax): multiply by 127/absmax, round, and the
    codes land in [-127, 127].  The quotient 127/absmax is one fp32 division;
    the product value * quotient is one fp32 multiplication.  absmax == 0
    yields code 0 (nothing to scale).  Returns int8.
    """
    x = np.asarray(values_f32, dtype=np.float32)
    a = np.asarray(absmax_f32, dtype=np.float32)[:, None]
    safe = np.where(a > 0, a, np.float32(1.0)).astype(np.float32)
    inv = (np.float32(Q_MAX) / safe).astype(np.float32)
    prod = (x * inv).astype(np.float32)
    q = np.clip(round_half_away(prod), -Q_MAX, Q_MAX)
    q = np.where(a > 0, q, 0.0)
    return q.astype(np.int8)


# ---------------------------------------------------------------------------
# a0: weight quantisation (done once, on ``.to(device)``)
# ---------------------------------------------------------------------------

def quantize_weight(W: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """W fp16 [N,K] -> (CB int8 [N,K], SCB fp32 [N]).

    One scale per output feature j ("column-wise for weights": the columns of
    W^T are the rows of the ``nn.Linear`` weight).  SCB[j] is the absmax of
    row j, so that ``CB * SCB / 127`` recovers W (page "Hugging Face
    integrates LLM.int8()", "Integration into transformers").
    """
    Wf = np.asarray(W, dtype=np.float16).astype(np.float32)
    SCB = np.abs(Wf).max(axis=1).astype(np.float32) if Wf.shape[1] else np.zeros(Wf.shape[0], np.float32)
    CB = absmax_codes(Wf, SCB)
    return CB, SCB


def dequantize_weight(CB: np.ndarray, SCB: np.ndarray) -> np.ndarray:
    """fp32 recovery ``(CB * SCB) / 127`` evaluated left to right in fp32."""
    prod = (CB.astype(np.float32) * SCB.astype(np.float32)[:, None]).astype(np.float32)
    return (prod / np.float32(Q_MAX)).astype(np.float32)


# ---------------------------------------------------------------------------
# a1/a2: column outliers and their ascending index list (``state.idx``)
# ---------------------------------------------------------------------------

def outlier_mask(X: np.ndarray, threshold: float) -> np.ndarray:
    """Boolean [K]: column k is an outlier iff some |X[t,k]| > threshold.

    ``threshold`` is taken as fp32 (the C boundary passes a float).  A
    non-positive threshold switches the decomposition off (empty set).
    NaN never compares greater, so a NaN entry never flags a column.
    """
    thr = np.float32(threshold)
    K = X.shape[1]
    if not thr > 0:
        return np.zeros(K, dtype=bool)
    ax = np.abs(np.asarray(X, dtype=np.float16).astype(np.float32))
    return (ax > thr).any(axis=0) if X.shape[0] else np.zeros(K, dtype=bool)


def outlier_index(mask: np.ndarray) -> np.ndarray:
    """Ascending int32 list of outlier columns (issue #1609 prints it sorted)."""
    return np.nonzero(mask)[0].astype(np.int32)


# ---------------------------------------------------------------------------
# a3/a4: row-wise activation quantisation and the fp16 outlier operands
# ---------------------------------------------------------------------------

def quantize_rows(X: np.ndarray, mask: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """X fp16 [T,K] -> (Xq int8 [T,K], sA fp32 [T]).

    "row-wise for activations": sA[t] is the absmax of row t over the
    non-outlier columns; those columns get absmax codes, outlier columns get
    code 0 (their contribution travels through the fp16 product instead).
    """
    Xf = np.asarray(X, dtype=np.float16).astype(np.float32)
    kept = np.where(mask[None, :], np.float32(0.0), np.abs(Xf)).astype(np.float32)
    sA = kept.max(axis=1).astype(np.float32) if Xf.shape[1] else np.zeros(Xf.shape[0], np.float32)
    Xq = absmax_codes(np.where(mask[None, :], np.float32(0.0), Xf), sA)
    Xq[:, mask] = 0
    return Xq, sA


def outlier_operands(X: np.ndarray, CB: np.ndarray, SCB: np.ndarray, idx: np.ndarray):
    """(Xo fp16 [T,n_out], Wo fp16 [N,n_out]) for the 16-bit outlier matmul.

    Xo gathers the outlier columns of X unchanged.  With has_fp16_weights=False
    the fp16 weight is gone, so Wo is recovered from CB/SCB as
    ``fp16((CB * SCB) / 127)`` at the outlier columns.
    """
    Xo = np.asarray(X, dtype=np.float16)[:, idx]
    Wo = dequantize_weight(CB[:, idx], SCB).astype(np.float16)
    return Xo, Wo


# ---------------------------------------------------------------------------
# a5: the int8 x int8 -> int32 product
# ---------------------------------------------------------------------------

def int8_matmul(Xq: np.ndarray, CB: np.ndarray) -> np.ndarray:
    """acc[t,j] = sum_k Xq[t,k] * CB[j,k], exact, returned as int32.

    |acc| <= K * 127**2, which fits int32 for K < 133144 and is far below
    2**53, so an fp64 matmul of the integer codes is exact in any order.
    """
    K = Xq.shape[1]
    assert K * Q_MAX * Q_MAX < 2**31, "int32 accumulator would overflow"
    acc = Xq.astype(np.float64) @ CB.astype(np.float64).T
    return acc.astype(np.int64).astype(np.int32)


# ---------------------------------------------------------------------------
# a7: dequantise, add the fp16 outlier product and the bias
# ---------------------------------------------------------------------------

def combine(acc, sA, SCB, Xo, Wo, bias) -> np.ndarray:
    """Y fp64 [T,N] = acc * sA[t] * SCB[j] / 127**2 + Xo @ Wo^T + bias.

    Step 3 of the method: the int8 result is scaled back with the row
    constant times the column constant, then summed with the 16-bit outlier
    product; the bias of ``nn.Linear`` is added last.
    """
    Y = acc.astype(np.float64) * sA.astype(np.float64)[:, None] * SCB.astype(np.float64)[None, :]
    Y = Y / float(Q_MAX * Q_MAX)
    if Xo.shape[1]:
        Y = Y + Xo.astype(np.float64) @ Wo.astype(np.float64).T
    if bias is not None:
        Y = Y + np.asarray(bias, dtype=np.float16).astype(np.float64)[None, :]
    return Y


def linear_forward(X, CB, SCB, bias, threshold, rows=None) -> dict:
    """Whole forward; returns every stage.

    ``rows`` (optional index array) restricts the per-row stages (a3-a7) to a
    subset of token rows.  The outlier set is always computed over all of X,
    because one token is enough to flag a column.
    """
    X = np.asarray(X, dtype=np.float16)
    mask = outlier_mask(X, threshold)
    idx = outlier_index(mask)
    Xs = X if rows is None else X[np.asarray(rows)]
    Xq, sA = quantize_rows(Xs, mask)
    Xo, Wo = outlier_operands(Xs, CB, SCB, idx)
    acc = int8_matmul(Xq, CB)
    Y = combine(acc, sA, SCB, Xo, Wo, bias)
    return {"mask": mask, "idx": idx, "n_out": int(idx.size), "Xq": Xq, "sA": sA,
            "Xo": Xo, "Wo": Wo, "acc": acc, "Y": Y}


def linear_forward_fp16w(X, W, bias, threshold, rows=None) -> dict:
    """Forward with has_fp16_weights=True: W stays fp16 and is quantised anew
    in every forward (bitsandbytes Linear8bitLt docstring, ``has_fp16_weights``).

    Reading taken: with the fp16 weight at hand, the outlier columns are
    multiplied with W's own fp16 values, Wo = W[:, idx], instead of the
    dequantised CB.
    """
    W = np.asarray(W, dtype=np.float16)
    X = np.asarray(X, dtype=np.float16)
    CB, SCB = quantize_weight(W)
    mask = outlier_mask(X, threshold)
    idx = outlier_index(mask)
    Xs = X if rows is None else X[np.asarray(rows)]
    Xq, sA = quantize_rows(Xs, mask)
    Xo = Xs[:, idx]
    Wo = W[:, idx]
    acc = int8_matmul(Xq, CB)
    Y = combine(acc, sA, SCB, Xo, Wo, bias)
    return {"mask": mask, "idx": idx, "n_out": int(idx.size), "Xq": Xq, "sA": sA, "CB": CB, "SCB": SCB,
            "Xo": Xo, "Wo": Wo, "acc": acc, "Y": Y}


# ---------------------------------------------------------------------------
# bf16 (the module is documented for "fp16 / bf16 weights"): numpy has no
# bfloat16 type, so bf16 values are carried as uint16 bit patterns -- the
# upper half of the fp32 pattern.
# ---------------------------------------------------------------------------

def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact widening: the bf16 pattern is the top 16 bits of the fp32 pattern."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 pattern, round to nearest, ties to even (NaN stays NaN)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    return np.where(nan, np.uint16(0x7FC0), rounded).astype(np.uint16)


def quantize_weight_bf16(W_u16: np.ndarray):
    """bf16 W [N,K] (patterns) -> (CB, SCB): the absmax rule of quantize_weight."""
    Wf = bf16_to_f32(W_u16)
    SCB = np.abs(Wf).max(axis=1).astype(np.float32) if Wf.shape[1] else np.zeros(Wf.shape[0], np.float32)
    return absmax_codes(Wf, SCB), SCB


def linear_forward_bf16(X_u16, CB, SCB, bias_u16, threshold, rows=None) -> dict:
    """The forward for bf16 activations / bias / output; outlier weights are
    bf16((CB * SCB) / 127).  Every step is the fp16 forward's step with bf16
    in place of fp16."""
    Xf = bf16_to_f32(X_u16)
    thr = np.float32(threshold)
    K = Xf.shape[1]
    mask = (np.abs(Xf) > thr).any(axis=0) if (thr > 0 and Xf.shape[0]) else np.zeros(K, bool)
    idx = outlier_index(mask)
    Xs = Xf if rows is None else Xf[np.asarray(rows)]
    kept = np.where(mask[None, :], np.float32(0.0), np.abs(Xs)).astype(np.float32)
    sA = kept.max(axis=1).astype(np.float32) if K else np.zeros(Xs.shape[0], np.float32)
    Xq = absmax_codes(np.where(mask[None, :], np.float32(0.0), Xs), sA)
    Xq[:, mask] = 0
    Xo = Xs[:, idx]                                                   # exact (bf16 values)
    Wo = bf16_to_f32(f32_to_bf16(dequantize_weight(CB[:, idx], SCB)))
    acc = int8_matmul(Xq, CB)
    bias = None if bias_u16 is None else bf16_to_f32(bias_u16)
    Y = acc.astype(np.float64) * sA.astype(np.float64)[:, None] * SCB.astype(np.float64)[None, :]
    Y = Y / float(Q_MAX * Q_MAX)
    if idx.size:
        Y = Y + Xo.astype(np.float64) @ Wo.astype(np.float64).T
    if bias is not None:
        Y = Y + bias.astype(np.float64)[None, :]
    return {"mask": mask, "idx": idx, "n_out": int(idx.size), "Xq": Xq, "sA": sA, "Xo": f32_to_bf16(Xo),
            "Wo": f32_to_bf16(Wo), "acc": acc, "Y": Y}


def linear_forward_fp16w_bf16(X_u16, W_u16, bias_u16, threshold, rows=None) -> dict:
    """has_fp16_weights=True with bf16 operands: W (bf16 patterns) is quantised
    in the forward, and the outlier columns are multiplied with W's own bf16
    columns W[:, idx] (the reading of linear_forward_fp16w, with bf16 in place
    of fp16)."""
    CB, SCB = quantize_weight_bf16(W_u16)
    r = linear_forward_bf16(X_u16, CB, SCB, None, threshold, rows)
    idx = r["idx"]
    Wo = bf16_to_f32(np.asarray(W_u16, dtype=np.uint16)[:, idx]).astype(np.float64)
    Xo = bf16_to_f32(r["Xo"]).astype(np.float64)
    Y = r["acc"].astype(np.float64) * r["sA"].astype(np.float64)[:, None] * SCB.astype(np.float64)[None, :]
    Y = Y / float(Q_MAX * Q_MAX)
    if idx.size:
        Y = Y + Xo @ Wo.T
    if bias_u16 is not None:
        Y = Y + bf16_to_f32(bias_u16).astype(np.float64)[None, :]
    r.update({"CB": CB, "SCB": SCB, "Wo": np.asarray(W_u16, dtype=np.uint16)[:, idx], "Y": Y})
    return r


def y_tolerance_bf16(Yref: np.ndarray) -> float:
    """Allowed max |Y - Yref| for a bf16 output: 2^-8 * max|Yref| + 2e-3.

    bf16 keeps 8 significant bits (7 stored), so rounding the fp32 result to
    the nearest bf16 can move it by up to 2^-8 |Y| (the unit roundoff).  The
    oracle multiplies the same bf16-rounded outlier weights as the kernel, so
    that output rounding is the only error of this size; the 2e-3 covers the
    kernel's fp32 accumulation."""
    return 2.0**-8 * float(np.abs(Yref).max(initial=0.0)) + 2e-3


def y_tolerance(Yref: np.ndarray) -> float:
    """Allowed max |Y - Yref| for the fp16 output: 1e-3 * max|Yref| + 2e-3."""
    return 1e-3 * float(np.abs(Yref).max(initial=0.0)) + 2e-3
