"""Plain CPU oracle for the LLM.int8() ``Linear8bitLt`` forward pass and its input gradient.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the test-suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, tables or helpers with the CUDA library and imports nothing from it.

Sources (the pages this restates; none of them prints code for these steps):

* "`bitsandbytes` - `Linear8bitLt` integration into `transformers` models"
  (HF transformers PR #17901), section "About the mixed quantization method in
  few words": operations on outlier features run in fp16, everything else in
  int8.
* "LLM.int8() Refactoring: Part 1" (bitsandbytes PR #1401), section
  "Improved kernels for inference": one fused kernel calibrates the activation
  scale and quantises (``int8_vectorwise_quant``); kernels work on row-major
  data.  Section "Deprecations": ``igemmlt`` becomes ``int8_linear_matmul``,
  ``mm_dequant`` becomes ``int8_mm_dequant``.  Section "Next steps": an int8
  dequantize op.  Review comment on ``bitsandbytes/autograd/_functions.py``:
  ``state.idx`` holds the outlier column indices of the activation.

The pages never write down the numeric rules.  The readings used here (each is
listed with its reason in the design notes of the repository):

* R1  row scale: ``SCA[i] = max |x[i, j]|`` over the elements of row i whose
      magnitude is below the threshold (all elements when threshold == 0);
      an empty maximum is 0.  Exclusion is per element.
* R2  outlier columns: ``O = {j : |x[i, j]| >= threshold for some i}`` when
      threshold > 0 ("at or above"); ``O`` is empty when threshold == 0.
* R3  codes: ``r = fl32(127 / SCA[i])`` (one IEEE fp32 division),
      ``q = clamp(rne(fl32(x * r)), -127, 127)``; 0 when SCA[i] == 0; and
      every column of ``O`` is 0 in every row (the fp16 path owns it).
* R4  weights use the same rule with threshold 0 (row-wise absmax ``SCB``).
* R5  ``C = CA . CB^T`` exactly, in integers.
* R6  ``out = fp16( C*SCA[i]*SCB[n]/127^2 + bias[n]
                   + (SCB[n]/127) * sum_{j in O} x[i,j]*CB[n,j] )``
      evaluated in float64 with one final round to fp16; the outlier weights
      are the int8 weights dequantised (the boundary takes no fp16 weight).
* R7  dequantize op: ``W = fp16(CB * SCB[n] / 127)``, one rounding.
* R9  input gradient (training through the frozen int8 layer):
      ``dX = fp16(dY . W^)`` evaluated in float64 with one final round, where
      ``W^ = dequant(CB, SCB)`` is the fp16 dequantised weight.  This is the
      chain rule for ``y = X . W^T + bias``; the pages only say that int8
      modules carry trainable adapters, so the layer must pass gradients on.

Precision: the quantisation decisions (R1-R4) are taken in IEEE fp32, the
precision the GPU takes them in; everything after the integer product is
float64.  Parity: every function here is pinned by ``tests/test_oracle_pins.py``
(closed-form cases, error bounds, invariants, brute force, special cases that
reduce to textbook formulas).
"""

from __future__ import annotations

import numpy as np

INT8_MAX = 127.0


def _as_f16(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype != np.float16:
        raise TypeError(f"expected float16 input, got {x.dtype}")
    return x


def quantize_rowwise(X, threshold: float = 0.0):
    """Fused row-wise absmax calibration + int8 quantisation + outlier detection.

    "LLM.int8() Refactoring: Part 1", section "Improved kernels for inference"
    (``int8_vectorwise_quant``), with readings R1-R3 of the module docstring.

    Args:
      X: float16 array [M, K] (row-major: tokens x features).
      threshold: outlier threshold (0 disables outlier handling).

    Returns:
      (CA int8 [M, K], SCA float32 [M], cols int64 [n_o] sorted ascending).
    """
    X = _as_f16(X)
    if X.ndim != 2:
        raise ValueError("X must be 2-D")
    tau = np.float32(threshold)
    if not np.isfinite(tau) or tau < 0:
        raise ValueError("threshold must be finite and >= 0")
    xf = X.astype(np.float32)                  # exact widening
    ax = np.abs(xf)

    # R2: outlier columns (any element at or above the threshold)
    if tau > 0:
        is_big = ax >= tau
        cols = np.flatnonzero(is_big.any(axis=0)).astype(np.int64)
        kept = np.where(is_big, np.float32(0), ax)
    else:
        cols = np.zeros(0, dtype=np.int64)
        kept = ax

    # R1: per-row absmax over the kept elements (0 for an empty row)
    if X.shape[1] == 0:
        SCA = np.zeros(X.shape[0], dtype=np.float32)
    else:
        SCA = kept.max(axis=1).astype(np.float32)

    # R3: one fp32 division per row, one fp32 multiply per element, RNE
    with np.errstate(divide="ignore"):
        r = np.where(SCA > 0, np.float32(INT8_MAX) / SCA, np.float32(0)).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        prod = (xf * r[:, None]).astype(np.float32)
    q = np.rint(prod)                          # round half to even
    q = np.clip(q, -INT8_MAX, INT8_MAX)
    CA = q.astype(np.int8)
    CA[:, cols] = 0
    return CA, SCA, cols


def quantize_weight_rowwise(W):
    """Row-wise int8 quantisation of an fp16 weight [N, K] -> (CB, SCB).

    "`bitsandbytes` - `Linear8bitLt` integration into `transformers` models"
    (``Int8Params`` keeps the int8 weight) and "LLM.int8() Refactoring: Part 1"
    (``CB`` in the review of ``_functions.py``): reading R4, threshold 0.
    """
    CB, SCB, _ = quantize_rowwise(W, 0.0)
    return CB, SCB


def outlier_bitmap(cols, K: int) -> np.ndarray:
    """Column set -> uint32 words, bit (j % 32) of word (j // 32) set for j in cols."""
    words = np.zeros((K + 31) // 32, dtype=np.uint32)
    for j in np.asarray(cols, dtype=np.int64):
        words[j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return words


def int8_linear_matmul(A, B) -> np.ndarray:
    """``C[i, n] = sum_k A[i, k] * B[n, k]`` exactly (reading R5).

    "LLM.int8() Refactoring: Part 1", section "Deprecations"
    (``igemmlt`` -> ``int8_linear_matmul``), row-major operands.

    The float64 product of int8-valued matrices is exact here: every partial
    sum is an integer of magnitude <= 127*127*K < 2**53.
    """
    A = np.asarray(A)
    B = np.asarray(B)
    if A.dtype != np.int8 or B.dtype != np.int8:
        raise TypeError("int8 operands expected")
    if A.shape[1] != B.shape[1]:
        raise ValueError("inner dimensions differ")
    K = A.shape[1]
    if 127 * 127 * K >= 2 ** 53:
        raise ValueError("K too large for an exact float64 product")
    Cd = A.astype(np.float64) @ B.astype(np.float64).T
    C = Cd.astype(np.int64)
    if C.size and (C.max() > np.iinfo(np.int32).max or C.min() < np.iinfo(np.int32).min):
        raise OverflowError("int32 accumulator overflow")
    return C.astype(np.int32)


def int8_mm_dequant(C, SCA, SCB, bias=None) -> np.ndarray:
    """``out = fp16(C * SCA[i] * SCB[n] / 127^2 + bias[n])`` in float64.

    "LLM.int8() Refactoring: Part 1", section "Deprecations"
    (``mm_dequant`` -> ``int8_mm_dequant``) and the commit "New naive
    mm_dequant kernel for row-major".
    """
    C = np.asarray(C).astype(np.float64)
    sa = np.asarray(SCA, dtype=np.float32).astype(np.float64)
    sb = np.asarray(SCB, dtype=np.float32).astype(np.float64)
    y = C * sa[:, None] * sb[None, :] / (INT8_MAX * INT8_MAX)
    if bias is not None:
        y = y + _as_f16(bias).astype(np.float64)[None, :]
    return y.astype(np.float16)


def dequant(CB, SCB) -> np.ndarray:
    """int8 dequantize op: ``W = fp16(CB * SCB[n] / 127)`` in float64 (reading R7).

    "LLM.int8() Refactoring: Part 1", section "Next steps"
    ("Add an int8 dequantize op").
    """
    CB = np.asarray(CB)
    if CB.dtype != np.int8:
        raise TypeError("CB must be int8")
    sb = np.asarray(SCB, dtype=np.float32).astype(np.float64)
    return (CB.astype(np.float64) * sb[:, None] / INT8_MAX).astype(np.float16)


def _forward_f64(X, CB, SCB, bias, threshold, rows=None):
    """Un-rounded float64 forward value for the selected rows (all by default)."""
    X = _as_f16(X)
    CA, SCA, cols = quantize_rowwise(X, threshold)   # O is a union over ALL rows
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        CA, SCA, Xs = CA[rows], SCA[rows], X[rows]
    else:
        Xs = X
    C = int8_linear_matmul(CA, CB).astype(np.float64)
    sa = SCA.astype(np.float64)
    sb = np.asarray(SCB, dtype=np.float32).astype(np.float64)
    y = C * sa[:, None] * sb[None, :] / (INT8_MAX * INT8_MAX)
    if cols.size:
        # fp16 outlier sub-GEMM against the dequantised int8 weight columns
        xo = Xs[:, cols].astype(np.float64)
        wo = CB[:, cols].astype(np.float64)
        y = y + (xo @ wo.T) * (sb[None, :] / INT8_MAX)
    if bias is not None:
        y = y + _as_f16(bias).astype(np.float64)[None, :]
    return y


def linear8bit_forward(X, CB, SCB, bias=None, threshold: float = 6.0, rows=None):
    """LLM.int8() mixed-decomposition linear forward (readings R1-R6).

    "`bitsandbytes` - `Linear8bitLt` integration into `transformers` models",
    section "About the mixed quantization method in few words", composed with
    the three ops of "LLM.int8() Refactoring: Part 1" (quantise, int8 matmul,
    dequant) plus the fp16 outlier product.

    Args:
      X: fp16 [M, K]; CB: int8 [N, K]; SCB: fp32 [N]; bias: fp16 [N] or None.
      rows: optional row subset to evaluate (quantisation still sees all rows,
        since the outlier set is a union over rows).

    Returns fp16 [M or len(rows), N].
    """
    return _forward_f64(X, CB, SCB, bias, threshold, rows).astype(np.float16)


def linear8bit_backward_input(dY, CB, SCB, rows=None):
    """Input gradient of the int8 linear layer (reading R9).

    "`bitsandbytes` - `Linear8bitLt` integration into `transformers` models",
    discussion of fine-tuning: trainable adapters sit on top of frozen int8
    modules, so the gradient reaches the layer input through the dequantised
    weight ``W^ = dequant(CB, SCB)``; the int8 weight gets no gradient.

    Args:
      dY: fp16 [M, N] gradient of the layer output; CB: int8 [N, K]; SCB: fp32 [N].
      rows: optional row subset of dY to evaluate.

    Returns fp16 [M or len(rows), K] = fp16(dY . W^) (float64 product, one rounding).
    """
    dY = _as_f16(dY)
    if rows is not None:
        dY = dY[np.asarray(rows, dtype=np.int64)]
    W = dequant(CB, SCB).astype(np.float64)
    return (dY.astype(np.float64) @ W).astype(np.float16)
