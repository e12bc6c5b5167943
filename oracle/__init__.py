"""CPU oracle for the LLM.int8() forward linear layer.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  Nothing in the product package
imports it, and it imports nothing from the product package.

Two restatements of the same steps, pinned by the same tests and checked to
agree bit for bit on every integer stage: ``llm_int8`` (numpy; its int8
product is an fp64 matmul of small integers, exact) and ``cpp`` (plain C++17
loops in ``llm_int8_ref.cpp``, built with g++ by ``cpp.build()``; the CPU
baseline ``bench.py`` times).
"""

from .llm_int8 import (  # noqa: F401
    Q_MAX,
    absmax_codes,
    combine,
    dequantize_weight,
    int8_matmul,
    linear_forward,
    linear_forward_fp16w,
    bf16_to_f32,
    f32_to_bf16,
    quantize_weight_bf16,
    linear_forward_bf16,
    linear_forward_fp16w_bf16,
    y_tolerance_bf16,
    outlier_index,
    outlier_mask,
    outlier_operands,
    quantize_rows,
    quantize_weight,
    round_half_away,
    y_tolerance,
)
