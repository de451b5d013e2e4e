"""LLM.int8() Linear8bitLt forward for B200 (sm_100a).

The compute path is the CUDA library ``libi8lt.so`` (C ABI in
``include/i8lt.h``); this package is a thin ctypes binding over it with the
same entry-point names.  PyTorch supplies device memory and streams only.
"""

from ._binding import (  # noqa: F401
    I8Error,
    LIB_PATH,
    STATUS,
    i8_dequant,
    i8_dequant_transposed,
    i8_gather_column_blocks,
    i8_int8_linear_matmul,
    i8_int8_linear_matmul_ws,
    i8_int8_mm_dequant,
    i8_linear8bit_backward_input,
    i8_linear8bit_forward,
    i8_linear8bit_forward_multi,
    i8_linear8bit_forward_static,
    i8_linear8bit_matmul_dequant,
    i8_linear8bit_multi_workspace_size,
    i8_linear8bit_prepare,
    i8_linear8bit_workspace_layout,
    i8_linear8bit_workspace_size,
    i8_nf4_dequant,
    i8_nf4_gemv,
    i8_nf4_levels,
    i8_nf4_quantize,
    i8_outlier_columns,
    i8_quantize_rowwise,
    i8_read_status,
    i8_selftest_bounded_wait,
    lib,
)
from .layer import Linear8bitLt  # noqa: F401
