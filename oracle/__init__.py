"""CPU oracle for the LLM.int8() forward linear layer.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  Nothing in the product package
imports it, and it imports nothing from the product package.
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
