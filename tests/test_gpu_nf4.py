"""GPU parity of the 4-bit NF4 weight-only product against oracle/nf4.py.

Bit-exact: the packed codes, the block scales and the fp16 dequantised weight.
The product: |gpu - oracle| <= (64 + K/512) * 2^-23 * sum_k |x_k * w_k| + one fp16
ulp of the oracle value, a bound derived from the kernel's fp32 evaluation: per row,
token and half block two 16-term fused multiply-add chains and their sum, one scaled
accumulation per half block (at most K/256 per lane), a 3-level sum over the 8 lanes
of a row and at most 7 additions of cluster partial sums -- fewer than 64 + K/512
roundings of size 2^-24 relative to the running sums, each bounded by the sum of
magnitudes -- then one rounding to fp16 on each side.
"""

import numpy as np
import pytest
import torch

from oracle import nf4
from int8_mixed_precision_vectorwise_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def i8():
    from int8_mixed_precision_vectorwise_b200 import build
    build.build()
    import int8_mixed_precision_vectorwise_b200 as m
    m.lib()
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def check_gemv(got, X, packed, absmax, what):
    ref = nf4.nf4_gemv(X, packed, absmax).astype(np.float64)
    mag = np.abs(X.astype(np.float64)) @ np.abs(nf4.nf4_weight_exact(packed, absmax)).T
    K = X.shape[1]
    bound = (64 + K / 512) * 2.0 ** -23 * mag + np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(err <= bound), f"{what}: {int((err > bound).sum())} out of bound, max err {err.max():.3g}"


@pytest.mark.parametrize("N,K", [(1, 64), (40, 192), (300, 4160), (4096, 4096), (33, 8256)])
def test_quantize_and_dequant_bit_exact(i8, N, K):
    W = wl.weight(700 + N, N, K)
    W[0, :64] = np.float16(0)                                   # a zero block
    if N > 1:
        W[1, 64:128] = np.linspace(-1, 1, 64).astype(np.float16)  # exact block extremes
    packed, absmax = i8.i8_nf4_quantize(dev(W))
    rp, ra = nf4.quantize_nf4(W)
    assert np.array_equal(host(absmax).view(np.uint32), ra.view(np.uint32))
    assert np.array_equal(host(packed), rp)
    Wh = i8.i8_nf4_dequant(packed, absmax)
    assert np.array_equal(host(Wh).view(np.uint16), nf4.dequant_nf4(rp, ra).view(np.uint16))


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("N,K", [(100, 128), (1000, 8256), (4096, 4096), (257, 16384)])
def test_gemv_against_oracle(i8, M, N, K):
    W = wl.weight(710 + N, N, K)
    X, _ = wl.activation(wl.BASE_SEED + 711 + M, M, K, 2, (8.0, 30.0))
    rp, ra = nf4.quantize_nf4(W)
    out = host(i8.i8_nf4_gemv(dev(X), dev(rp), dev(ra)))
    check_gemv(out, X, rp, ra, f"M={M} N={N} K={K}")


# Shapes for which the launcher picks each kind of work split: K split over clusters
# of 1, 2, 3, 4, 6 and 8 CTAs, 32 / 64 / 128 rows per CTA, every token-slot width,
# ragged N and K (not multiples of the rows per CTA or of 256 weights).
@pytest.mark.parametrize("M,N,K", [(3, 96, 576), (1, 96, 1088), (6, 1500, 2112), (2, 96, 2112),
                                   (3, 3000, 2112), (1, 96, 3136), (6, 96, 4160), (7, 200, 4160),
                                   (2, 4100, 6208), (1, 130, 64), (8, 33, 320)])
def test_gemv_work_splits(i8, M, N, K):
    W = wl.weight(740 + N, N, K)
    X, _ = wl.activation(wl.BASE_SEED + 741 + M, M, K, 3, (8.0, 30.0))
    rp, ra = nf4.quantize_nf4(W)
    out = host(i8.i8_nf4_gemv(dev(X), dev(rp), dev(ra)))
    check_gemv(out, X, rp, ra, f"M={M} N={N} K={K}")


@pytest.mark.parametrize("N,K", [(28672, 8192), (8192, 28672)])
@pytest.mark.parametrize("M", [1, 4, 8])
def test_gemv_llama70b_sampled_rows(i8, M, N, K):
    """The Llama-70B FFN shapes the bench streams: the GPU quantises and multiplies the whole
    weight; codes, scales and outputs are compared on 256 sampled weight rows (quantisation
    and the product are row by row, so the sample is checked exactly as in the whole)."""
    W = wl.weight(720 + N, N, K)
    X, _ = wl.activation(wl.BASE_SEED + 721 + M, M, K, 8, (30.0, 30.0))
    packed, absmax = i8.i8_nf4_quantize(dev(W))
    out = host(i8.i8_nf4_gemv(dev(X), packed, absmax))
    rows = np.sort(np.random.default_rng(N + M).choice(N, 256, replace=False))
    rp, ra = nf4.quantize_nf4(W[rows])
    assert np.array_equal(host(packed)[rows], rp)
    assert np.array_equal(host(absmax)[rows].view(np.uint32), ra.view(np.uint32))
    check_gemv(out[:, rows], X, rp, ra, f"llama70b M={M} {N}x{K}")


def test_gemv_repeat_is_deterministic(i8):
    W = wl.weight(730, 512, 2048)
    X, _ = wl.activation(wl.BASE_SEED + 731, 3, 2048, 1, (8.0, 30.0))
    packed, absmax = i8.i8_nf4_quantize(dev(W))
    a = i8.i8_nf4_gemv(dev(X), packed, absmax)
    b = i8.i8_nf4_gemv(dev(X), packed, absmax)
    assert torch.equal(a, b)
    # a K split over a cluster adds its partial sums in a fixed order too
    W = wl.weight(732, 8192, 28672)
    X, _ = wl.activation(wl.BASE_SEED + 733, 8, 28672, 4, (8.0, 30.0))
    packed, absmax = i8.i8_nf4_quantize(dev(W))
    a = i8.i8_nf4_gemv(dev(X), packed, absmax)
    b = i8.i8_nf4_gemv(dev(X), packed, absmax)
    assert torch.equal(a, b)
