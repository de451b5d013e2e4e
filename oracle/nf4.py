"""Plain CPU oracle for the 4-bit NF4 weight-only decode product (blocksize 64).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use it.  It shares
no code, tables or constant generators with the CUDA library.

Source: "Loading an LLM in 4 bits using bitsandbytes" (the Medium page), sections
"Normalized Float" and "Double Quantization": nf4 is a 4-bit type whose values
"were optimized for saving normally distributed variables"; weights are quantised
in blocks of 64, each block keeping a 32-bit scaling factor; the product is
computed in a separate compute dtype after dequantisation
(``bnb_4bit_compute_dtype``).  The page prints neither the 16 values nor the
rounding rule; the readings taken here (listed with their reasons in the design
notes):

* R11 levels: the NormalFloat construction.  With Q the standard normal quantile
      function and p* = 1 - (1/32 + 1/30) / 2, the positive levels are
      Q(1/2 + i (p* - 1/2) / 8) / Q(p*) for i = 1..8, the negative levels
      -Q(1/2 + i (p* - 1/2) / 7) / Q(p*) for i = 1..7, and 0: equal steps in
      probability on each half of N(0, 1), an exact zero, endpoints -1 and +1.
      Evaluated in float64, stored as fp32, ascending: code 7 is 0.
* R12 quantisation: blocks of 64 consecutive elements of the row-major weight
      (K % 64 == 0, so a block never straddles two rows); absmax = max |w| in
      fp32; y = fl32(w / absmax) (0 when absmax = 0); code = the number of
      midpoints m_i = fl32((v_i + v_{i+1}) / 2) strictly below y, i.e. the
      nearest level with ties to the lower one.  Byte j of a row holds the codes
      of elements 2j (low nibble) and 2j + 1 (high nibble).
* R13 dequantisation op (the weight handed back in fp16): W^ = fp16(fl32(v[code] * absmax)).
* R14 product: out[t, n] = fp16(sum_k X[t, k] * v[code[n, k]] * absmax[n, k / 64]),
      evaluated in float64 with one rounding: the dequantised weight enters the
      product exactly (the compute dtype of the page concerns how a library
      evaluates it; any evaluation in fp32 or wider is within the bound the tests
      derive).
      (Double quantisation of the scales is a storage option of the page, not
      part of this product, and is not built.)
"""

from __future__ import annotations

import numpy as np
from scipy.stats import norm

BLOCK = 64
P_STAR = 1.0 - (1.0 / 32.0 + 1.0 / 30.0) / 2.0


def nf4_levels() -> np.ndarray:
    """The 16 NF4 values (reading R11), fp32, ascending."""
    top = norm.ppf(P_STAR)
    pos = [norm.ppf(0.5 + i * (P_STAR - 0.5) / 8) / top for i in range(1, 9)]
    neg = [-norm.ppf(0.5 + i * (P_STAR - 0.5) / 7) / top for i in range(1, 8)]
    return np.array(sorted(neg + [0.0] + pos), dtype=np.float64).astype(np.float32)


def nf4_midpoints(levels=None) -> np.ndarray:
    """fl32((v_i + v_{i+1}) / 2), i = 0..14: the decision points of R12."""
    v = nf4_levels() if levels is None else np.asarray(levels, np.float32)
    return ((v[:-1] + v[1:]) / np.float32(2)).astype(np.float32)


def quantize_nf4(W):
    """Blockwise NF4 quantisation of an fp16 weight [N, K] (reading R12).

    Returns (packed uint8 [N, K/2], absmax fp32 [N, K/64])."""
    W = np.asarray(W)
    if W.dtype != np.float16 or W.ndim != 2:
        raise TypeError("fp16 [N, K] weight expected")
    N, K = W.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 64")
    w = W.astype(np.float32).reshape(N, K // BLOCK, BLOCK)
    absmax = np.abs(w).max(axis=2).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(absmax[..., None] > 0, w / absmax[..., None], np.float32(0)).astype(np.float32)
    mids = nf4_midpoints()
    codes = (y[..., None] > mids).sum(axis=-1).astype(np.uint8).reshape(N, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, absmax


def unpack_codes(packed) -> np.ndarray:
    """uint8 [N, K/2] -> codes uint8 [N, K] (element 2j low nibble, 2j + 1 high)."""
    p = np.asarray(packed, np.uint8)
    N, H = p.shape
    codes = np.empty((N, 2 * H), np.uint8)
    codes[:, 0::2] = p & 0x0F
    codes[:, 1::2] = p >> 4
    return codes


def dequant_nf4(packed, absmax) -> np.ndarray:
    """W^ = fp16(fl32(v[code] * absmax)) (reading R13), fp16 [N, K]."""
    codes = unpack_codes(packed)
    N, K = codes.shape
    v = nf4_levels()[codes].reshape(N, K // BLOCK, BLOCK)
    prod = (v * np.asarray(absmax, np.float32)[..., None]).astype(np.float32)
    return prod.reshape(N, K).astype(np.float16)


def nf4_weight_exact(packed, absmax) -> np.ndarray:
    """v[code] * absmax in float64 (exact: a product of two fp32 values), [N, K]."""
    codes = unpack_codes(packed)
    N, K = codes.shape
    v = nf4_levels().astype(np.float64)[codes].reshape(N, K // BLOCK, BLOCK)
    return (v * np.asarray(absmax, np.float32).astype(np.float64)[..., None]).reshape(N, K)


def nf4_gemv(X, packed, absmax) -> np.ndarray:
    """out = fp16(X . (v * absmax)^T) in float64 with one rounding (reading R14): X fp16 [M, K]."""
    X = np.asarray(X)
    if X.dtype != np.float16:
        raise TypeError("fp16 X expected")
    return (X.astype(np.float64) @ nf4_weight_exact(packed, absmax).T).astype(np.float16)
