"""CPU oracle for the LLM.int8() linear forward and the NF4 weight-only decode
product (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package; the product path never does.  ``oracle.nf4`` holds the
4-bit NF4 part.
"""
from .llm_int8 import (  # noqa: F401
    quantize_rowwise,
    quantize_weight_rowwise,
    outlier_bitmap,
    int8_linear_matmul,
    int8_mm_dequant,
    dequant,
    linear8bit_forward,
    linear8bit_backward_input,
)
