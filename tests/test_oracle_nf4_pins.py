"""Pins of the NF4 oracle (oracle/nf4.py) against what the definitions fix, on CPU.

Each pin is chosen so that a plausible mistake fails it: a wrong step count or
offset in the levels (checked through the normal CDF, the inverse of the quantile
function the oracle uses), a rounding rule that is not "nearest, ties to the
lower level" (exact rational brute force), a swapped nibble order, a dropped
block scale, a transposed product.
"""

from fractions import Fraction

import numpy as np
import pytest
from scipy.stats import norm

from oracle import nf4


def test_levels_structure():
    v = nf4.nf4_levels()
    assert v.dtype == np.float32 and v.shape == (16,)
    assert np.all(np.diff(v) > 0)
    assert v[7] == 0.0 and v[0] == -1.0 and v[15] == 1.0
    assert (v < 0).sum() == 7 and (v > 0).sum() == 8


def test_levels_are_equal_probability_steps_of_the_normal():
    """Positive level i sits at probability 1/2 + i (p* - 1/2) / 8 of N(0, 1) once scaled back
    by Q(p*); negative level -i at 1/2 + i (p* - 1/2) / 7 (mirror image)."""
    v = nf4.nf4_levels().astype(np.float64)
    top = norm.ppf(nf4.P_STAR)
    for i in range(1, 9):
        assert norm.cdf(v[7 + i] * top) == pytest.approx(0.5 + i * (nf4.P_STAR - 0.5) / 8, abs=2e-7)
    for i in range(1, 8):
        assert norm.cdf(-v[7 - i] * top) == pytest.approx(0.5 + i * (nf4.P_STAR - 0.5) / 7, abs=2e-7)


def _nearest_exact(y, levels):
    """Nearest level to y by exact rational distances, ties to the lower level."""
    fy = Fraction(float(y))
    best, bd = None, None
    for i, lv in enumerate(levels):
        d = abs(fy - Fraction(float(lv)))
        if bd is None or d < bd:
            best, bd = i, d
    return best


def test_quantize_is_nearest_level_brute_force():
    rng = np.random.default_rng(0)
    levels = nf4.nf4_levels()
    W = (rng.standard_normal((6, 128)) * 0.03).astype(np.float16)
    W[0, :64] = np.float16(0)                      # a zero block
    W[1, :8] = [0.5, -0.5, 0.25, -0.25, 0.125, 0.0, 0.75, -1.0]   # exact fractions of the block max
    W[1, 8:64] = np.float16(0)
    packed, absmax = nf4.quantize_nf4(W)
    codes = nf4.unpack_codes(packed)
    for n in range(W.shape[0]):
        for b in range(2):
            a = np.float32(np.abs(W[n, 64 * b:64 * (b + 1)].astype(np.float32)).max())
            assert absmax[n, b] == a
            for k in range(64 * b, 64 * (b + 1)):
                y = np.float32(0) if a == 0 else np.float32(np.float32(W[n, k]) / a)
                assert codes[n, k] == _nearest_exact(y, levels), (n, k, float(y))


def test_zero_block_and_extremes():
    W = np.zeros((1, 64), np.float16)
    W[0, 3] = np.float16(2.0)
    W[0, 5] = np.float16(-2.0)
    packed, absmax = nf4.quantize_nf4(W)
    codes = nf4.unpack_codes(packed)[0]
    assert absmax[0, 0] == 2.0
    assert codes[3] == 15 and codes[5] == 0 and codes[0] == 7
    Z = np.zeros((2, 128), np.float16)
    pz, az = nf4.quantize_nf4(Z)
    assert np.all(az == 0) and np.all(nf4.unpack_codes(pz) == 7) and np.all(nf4.dequant_nf4(pz, az) == 0)


def test_nibble_order():
    """Element 2j is the low nibble of byte j, element 2j + 1 the high nibble."""
    W = np.zeros((1, 64), np.float16)
    W[0, 0], W[0, 1], W[0, 2] = 1.0, -1.0, 0.0
    packed, _ = nf4.quantize_nf4(W)
    assert packed[0, 0] == 0x0F          # codes 15 (low), 0 (high)
    assert packed[0, 1] == 0x77          # codes 7, 7


def test_dequant_round_trip_bound():
    """|w - W^| <= absmax * (largest half gap between levels) + the fp16 and fp32 roundings."""
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float16)
    packed, absmax = nf4.quantize_nf4(W)
    Wh = nf4.dequant_nf4(packed, absmax).astype(np.float64)
    gap = np.diff(nf4.nf4_levels().astype(np.float64)).max() / 2
    a = np.repeat(absmax.astype(np.float64), 64, axis=1)
    err = np.abs(W.astype(np.float64) - Wh)
    assert np.all(err <= a * gap * (1 + 1e-6) + np.spacing(np.abs(Wh).astype(np.float16)).astype(np.float64))


def test_block_scale_applies_per_block():
    """The same codes in two blocks with different maxima dequantise to values in the ratio of
    the maxima (a dropped or shared block scale fails this)."""
    base = np.linspace(-1, 1, 64).astype(np.float16)
    W = np.concatenate([base * np.float16(0.5), base * np.float16(2.0)])[None, :].astype(np.float16)
    packed, absmax = nf4.quantize_nf4(W)
    c = nf4.unpack_codes(packed)[0]
    assert np.array_equal(c[:64], c[64:])
    assert absmax[0, 1] == 4 * absmax[0, 0]
    Wh = nf4.dequant_nf4(packed, absmax).astype(np.float64)[0]
    assert np.allclose(Wh[64:], 4 * Wh[:64], rtol=2e-3, atol=0)


def test_gemv_one_hot_selects_weight_columns():
    """A one-hot row of X picks one column of the dequantised weight (to the last fp16 bit,
    which the dequant op may round differently as it passes through fp32 first)."""
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((40, 192)) * 0.02).astype(np.float16)
    packed, absmax = nf4.quantize_nf4(W)
    Wh = nf4.dequant_nf4(packed, absmax)
    X = np.zeros((3, 192), np.float16)
    X[0, 5] = 1.0
    X[1, 130] = 1.0
    X[2, 191] = -1.0
    out = nf4.nf4_gemv(X, packed, absmax)
    assert out.shape == (3, 40)                      # [M, N]: a transposed product fails
    ulp = np.spacing(np.abs(Wh).astype(np.float16)).astype(np.float64)
    for row, col, sgn in ((0, 5, 1), (1, 130, 1), (2, 191, -1)):
        assert np.all(np.abs(out[row].astype(np.float64) - sgn * Wh[:, col].astype(np.float64)) <= ulp[:, col])


def test_gemv_hand_worked():
    """Weights on the levels 0 and +-1 of a block with max 1: W^ is W itself, so the product is
    a small integer dot product."""
    W = np.zeros((2, 64), np.float16)
    W[0, :4] = [1, -1, 1, 0]
    W[1, :4] = [0, 1, 1, -1]
    X = np.zeros((1, 64), np.float16)
    X[0, :4] = [3, 2, 1, 5]
    packed, absmax = nf4.quantize_nf4(W)
    out = nf4.nf4_gemv(X, packed, absmax)
    assert out.tolist() == [[2.0, -2.0]]             # 3 - 2 + 1 ; 2 + 1 - 5
