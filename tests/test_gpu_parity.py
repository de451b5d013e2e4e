"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bit-exact: int8 codes, fp32 absmax scales, outlier bitmaps / column lists and
int32 accumulators.  fp16 outputs: |gpu - oracle| <= 1e-2 + 1e-3 * |oracle|
element by element (the allclose form; 1e-2 alone would reject legitimate one-
ulp fp16 differences above 16, 1e-3 alone would reject them near 0).
Every oracle input is generated here or by the oracle itself; nothing the CUDA
path computed is ever fed to the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
from int8_mixed_precision_vectorwise_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 1e-3


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


def assert_close(got, ref, what=""):
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape
    d = np.abs(g - r)
    bad = d > ATOL + RTOL * np.abs(r)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} out of tolerance; first {tuple(i)} "
                             f"got {g[tuple(i)]} want {r[tuple(i)]}; max abs {d.max():.3g}")


def bitmap_np(t):
    return host(t).view(np.uint32)


def act(M, K, n_out, mag=(20.0, 60.0), seed=0):
    return wl.activation(wl.BASE_SEED + seed, M, K, n_out, mag)


# ------------------------------------------------------------------ quantise
QSHAPES = [
    (1, 16, 0.0, 0), (3, 1024, 6.0, 2), (37, 4096, 6.0, 4), (130, 5120, 6.0, 5), (64, 8192, 6.0, 8),
    (16, 11008, 6.0, 11), (5, 28672, 6.0, 8), (3, 40000, 6.0, 3), (300, 2064, 0.0, 0), (1000, 272, 6.0, 1),
    (9, 4096, 6.0, 0), (257, 1040, 2.5, 0),
    # enough rows for the ring-fed kernel (one CTA per SM, rows bulk-copied into shared memory)
    (4099, 4096, 6.0, 9),     # 2 rows per stage, an odd number of rows
    (2500, 1040, 6.0, 3),     # 2 rows per stage, short rows
    (1300, 8192, 6.0, 12),    # 1 row per stage
    (700, 11008, 0.0, 0),     # 6 vectors per thread, threshold 0
    (600, 16384, 6.0, 5),     # 8 vectors per thread, 4 stages
]


@pytest.mark.parametrize("M,K,tau,n_out", QSHAPES)
def test_quantize_rowwise_bit_exact(i8, M, K, tau, n_out):
    X, _ = act(M, K, n_out, seed=M + K)
    CA, SCA, bm = i8.i8_quantize_rowwise(dev(X), tau)
    rCA, rSCA, rcols = oracle.quantize_rowwise(X, tau)
    assert np.array_equal(host(CA), rCA)
    assert np.array_equal(host(SCA).view(np.uint32), rSCA.view(np.uint32))
    if tau > 0:
        assert np.array_equal(bitmap_np(bm), oracle.outlier_bitmap(rcols, K))


def test_quantize_edge_values(i8):
    """Exact threshold hits, just-below values, zero rows, rows of outliers only, fp16 extremes."""
    M, K = 8, 64
    X = np.zeros((M, K), np.float16)
    X[0, :] = 1.0
    X[0, 3] = 6.0                     # exactly at the threshold -> outlier column 3
    X[1, :] = np.float16(5.99609375)  # just below: no outlier
    X[2, :] = 0.0                     # zero row
    X[3, :] = 7.0                     # every column an outlier in this row
    X[4, :] = np.float16(65504.0)     # fp16 max
    X[4, 1::2] = -np.float16(0.5)
    X[5, :] = np.float16(6e-8)        # subnormal
    X[6, ::3] = np.float16(-2.5)
    X[7, :] = np.float16(1.5)
    X[7, 10] = np.float16(-1.5)
    for tau in (0.0, 6.0, 0.25):
        CA, SCA, bm = i8.i8_quantize_rowwise(dev(X), tau)
        rCA, rSCA, rcols = oracle.quantize_rowwise(X, tau)
        assert np.array_equal(host(CA), rCA), tau
        assert np.array_equal(host(SCA).view(np.uint32), rSCA.view(np.uint32)), tau
        if tau > 0:
            assert np.array_equal(bitmap_np(bm), oracle.outlier_bitmap(rcols, K))


@pytest.mark.parametrize("K,n_out,cap", [(4096, 4, 64), (11008, 11, 8), (64, 64, 64), (28672, 0, 16)])
def test_outlier_columns(i8, K, n_out, cap):
    X, _ = act(4, K, n_out, seed=K)
    _, _, bm = i8.i8_quantize_rowwise(dev(X), 6.0)
    idx, cnt = i8.i8_outlier_columns(bm, K, cap)
    _, _, rcols = oracle.quantize_rowwise(X, 6.0)
    assert int(host(cnt)[0]) == len(rcols)
    k = min(cap, len(rcols))
    assert host(idx)[:k].tolist() == rcols[:k].tolist()


def test_weight_quant_matches_oracle(i8):
    W = wl.weight(99, 520, 1040)
    CB, SCB, _ = i8.i8_quantize_rowwise(dev(W), 0.0)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    assert np.array_equal(host(CB), rCB)
    assert np.array_equal(host(SCB).view(np.uint32), rSCB.view(np.uint32))


# ------------------------------------------------------------------ int8 GEMM
# Tile schedules on 148 SMs (74 CTA pairs, 256 x 256 tiles): up to 37 tiles run
# as half tiles only; (4096, 4096) and (2048, 5120) end with a round of half
# tiles; (1792, 4864) and (2304, 4096) leave too many tiles for that and run
# whole tiles only.
GSHAPES = [(128, 256, 128), (1, 1, 16), (37, 300, 272), (300, 520, 1040), (256, 512, 4096), (513, 257, 160),
           (129, 1000, 2064), (16, 4096, 28672), (1024, 768, 512), (4096, 4096, 256), (2048, 5120, 256),
           (1792, 4864, 128), (2304, 4096, 144)]


@pytest.mark.parametrize("M,N,K", GSHAPES)
def test_int8_linear_matmul_bit_exact(i8, M, N, K):
    g = np.random.default_rng(M * 7 + N * 3 + K)
    A = g.integers(-128, 128, size=(M, K), dtype=np.int8)
    B = g.integers(-128, 128, size=(N, K), dtype=np.int8)
    A[0, :] = -128
    B[0, :] = -128
    C = i8.i8_int8_linear_matmul(dev(A), dev(B))
    assert np.array_equal(host(C), oracle.int8_linear_matmul(A, B))


def test_int8_linear_matmul_repeat_and_stream(i8):
    g = np.random.default_rng(1)
    A = g.integers(-127, 128, size=(384, 1024), dtype=np.int8)
    B = g.integers(-127, 128, size=(640, 1024), dtype=np.int8)
    ref = oracle.int8_linear_matmul(A, B)
    s = torch.cuda.Stream()
    dA, dB = dev(A), dev(B)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        outs = [i8.i8_int8_linear_matmul(dA, dB) for _ in range(3)]
    s.synchronize()
    for C in outs:
        assert np.array_equal(C.cpu().numpy(), ref)


# ------------------------------------------------------------------ dequant ops
@pytest.mark.parametrize("M,N,bias", [(7, 12, True), (33, 1001, False), (256, 4096, True), (1, 3, True)])
def test_mm_dequant(i8, M, N, bias):
    g = np.random.default_rng(M + N)
    C = g.integers(-2_000_000, 2_000_000, size=(M, N), dtype=np.int32)
    SCA = g.uniform(0.5, 8, size=M).astype(np.float32)
    SCB = g.uniform(0.01, 0.2, size=N).astype(np.float32)
    b = (g.standard_normal(N) * 0.01).astype(np.float16) if bias else None
    out = i8.i8_int8_mm_dequant(dev(C), dev(SCA), dev(SCB), None if b is None else dev(b))
    assert_close(host(out), oracle.int8_mm_dequant(C, SCA, SCB, b), "mm_dequant")


@pytest.mark.parametrize("N,K", [(3, 16), (520, 1040), (4096, 4096)])
def test_dequant(i8, N, K):
    W = wl.weight(N + K, N, K)
    CB, SCB = oracle.quantize_weight_rowwise(W)
    Wg = i8.i8_dequant(dev(CB), dev(SCB))
    assert_close(host(Wg), oracle.dequant(CB, SCB), "dequant")


# ------------------------------------------------------------------ fused forward
def _forward_case(i8, M, N, K, n_out, tau, with_bias, cap=256, mag=(20.0, 60.0), seed=0):
    X, _ = act(M, K, n_out, mag, seed=seed + M + N + K)
    W = wl.weight(seed + 5, N, K)
    b = wl.bias(seed + 6, N) if with_bias else None
    CB, SCB, _ = i8.i8_quantize_rowwise(dev(W), 0.0)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    assert np.array_equal(host(CB), rCB)
    out, ws = i8.i8_linear8bit_forward(dev(X), CB, SCB, None if b is None else dev(b), tau,
                                       max_outlier_cols=cap)
    code, count = i8.i8_read_status(ws)
    ref = oracle.linear8bit_forward(X, rCB, rSCB, b, tau)
    _, _, rcols = oracle.quantize_rowwise(X, tau)
    return host(out), ref, code, count, len(rcols)


FSHAPES = [
    (16, 1024, 1024, 2, 6.0, True),      # the single-linear workload
    (1, 16, 16, 0, 6.0, False),
    (37, 300, 272, 3, 6.0, True),
    (130, 520, 1040, 5, 6.0, False),
    (256, 512, 4096, 4, 6.0, True),
    (300, 257, 160, 0, 0.0, True),
    (513, 700, 2048, 70, 6.0, True),     # two fp16 k-blocks of outliers
    (200, 384, 512, 3, 0.0, False),      # threshold 0: outlier columns stay on the int8 path
    (4, 28672, 8192, 8, 6.0, False),     # decode-shaped
    (300, 520, 1040, 7, 6.0, True),      # outlier operands: a partly filled 16-column group
    (256, 512, 2048, 13, 6.0, False),
    (257, 384, 1024, 17, 6.0, True),     # just past the warp-MMA limit: tensor-core outlier k-block
    (3, 300, 272, 3, 6.0, True),         # decode-shaped, K split unevenly over the preparation cluster
    (16, 2048, 4096, 40, 6.0, True),     # decode-shaped, outliers in every CTA's column range
    (4096, 4096, 512, 4, 6.0, True),     # whole tiles, then a round of half tiles
    (2048, 5120, 1024, 70, 6.0, False),  # the same with the fp16 outlier k-blocks
    (2304, 4096, 256, 5, 6.0, True),     # whole tiles only
]


@pytest.mark.parametrize("M,N,K,n_out,tau,with_bias", FSHAPES)
def test_linear8bit_forward(i8, M, N, K, n_out, tau, with_bias):
    out, ref, code, count, n_ref = _forward_case(i8, M, N, K, n_out, tau, with_bias)
    assert code == 0
    assert count == (n_ref if tau > 0 else 0)
    assert_close(out, ref, "forward")


@pytest.mark.parametrize("n_out", [5, 70])
def test_forward_large_capacity(i8, n_out):
    """A capacity above the default 256 (larger list and gathered-operand buffers)."""
    out, ref, code, count, n_ref = _forward_case(i8, 300, 520, 1040, n_out, 6.0, True, cap=512)
    assert code == 0 and count == n_ref
    assert_close(out, ref, "forward (capacity 512)")


@pytest.mark.parametrize("M", [64, 8])
def test_forward_all_columns_outliers(i8, M):
    """Threshold below every magnitude: the int8 path is empty and out is the fp16 path alone."""
    N, K = 256, 128
    X, _ = act(M, K, 0, seed=3)
    X[0] = np.where(np.abs(X[0]) < 1e-2, np.float16(0.5), X[0])
    out, ref, code, count, n_ref = None, None, None, None, None
    W = wl.weight(8, N, K)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    o, ws = i8.i8_linear8bit_forward(dev(X), dev(rCB), dev(rSCB), None, 1e-3, max_outlier_cols=K)
    code, count = i8.i8_read_status(ws)
    assert code == 0 and count == K
    assert_close(host(o), oracle.linear8bit_forward(X, rCB, rSCB, None, 1e-3), "all-outlier")


@pytest.mark.parametrize("M", [32, 4])
def test_forward_outlier_overflow_status(i8, M):
    N, K = 256, 512
    X, _ = act(M, K, 20, seed=4)
    W = wl.weight(9, N, K)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    _, ws = i8.i8_linear8bit_forward(dev(X), dev(rCB), dev(rSCB), None, 6.0, max_outlier_cols=8)
    code, count = i8.i8_read_status(ws)
    assert code == 6 and count == 20
    # the same workspace recovers on the next call with enough capacity
    o, ws = i8.i8_linear8bit_forward(dev(X), dev(rCB), dev(rSCB), None, 6.0, max_outlier_cols=64)
    assert i8.i8_read_status(ws) == (0, 20)
    assert_close(host(o), oracle.linear8bit_forward(X, rCB, rSCB, None, 6.0), "after overflow")


def test_forward_deterministic(i8):
    X, _ = act(300, 1024, 3, seed=5)
    W = wl.weight(10, 777, 1024)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    dX, dCB, dSCB = dev(X), dev(rCB), dev(rSCB)
    a, ws = i8.i8_linear8bit_forward(dX, dCB, dSCB, None, 6.0)
    b, _ = i8.i8_linear8bit_forward(dX, dCB, dSCB, None, 6.0, workspace=ws)
    assert torch.equal(a, b)


def test_opt_mlp_pair_chain(i8):
    """OPT-350m-shaped fc1 -> ReLU -> fc2, each side chained on its own results."""
    W = wl.workloads()["C2"]
    l1, l2 = W.layers
    X, _, W1, b1 = wl.layer_inputs(2, 0, l1)
    _, _, W2, b2 = wl.layer_inputs(2, 1, l2)
    rCB1, rSCB1 = oracle.quantize_weight_rowwise(W1)
    rCB2, rSCB2 = oracle.quantize_weight_rowwise(W2)
    h = oracle.linear8bit_forward(X, rCB1, rSCB1, b1, 6.0)
    h = np.maximum(h, np.float16(0))
    ref2 = oracle.linear8bit_forward(h, rCB2, rSCB2, b2, 6.0)
    CB1, SCB1, _ = i8.i8_quantize_rowwise(dev(W1), 0.0)
    CB2, SCB2, _ = i8.i8_quantize_rowwise(dev(W2), 0.0)
    o1, _ = i8.i8_linear8bit_forward(dev(X), CB1, SCB1, dev(b1), 6.0)
    assert_close(host(o1), oracle.linear8bit_forward(X, rCB1, rSCB1, b1, 6.0), "fc1")
    o2, _ = i8.i8_linear8bit_forward(torch.relu(o1).contiguous(), CB2, SCB2, dev(b2), 6.0)
    assert_close(host(o2), ref2, "fc2 chained")
    # fc2 on the oracle's own hidden state: codes are then bit-exact
    CA2, SCA2, _ = i8.i8_quantize_rowwise(dev(h), 6.0)
    rCA2, rSCA2, _ = oracle.quantize_rowwise(h, 6.0)
    assert np.array_equal(host(CA2), rCA2)
    o2b, _ = i8.i8_linear8bit_forward(dev(h), CB2, SCB2, dev(b2), 6.0)
    assert_close(host(o2b), ref2, "fc2 on oracle hidden")


def test_selftest_bounded_wait_times_out(i8):
    import time
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    i8.i8_selftest_bounded_wait(st, 50_000_000)   # 50 ms
    torch.cuda.synchronize()
    assert time.time() - t0 < 10
    assert int(st.item()) == 5   # I8_ERR_TIMEOUT, and the context is still usable:
    assert torch.ones(4, device="cuda").sum().item() == 4


# ------------------------------------------------------------------ one-launch small forward
SMALL_SHAPES = [
    # M, N, K, planted columns, threshold, bias   (all take the one-launch kernel; on 148 SMs
    # K is split over clusters of 8, 8, 2, 4, 8, 8, 1 and 8 CTAs)
    (16, 1024, 1024, 2, 6.0, True),     # the single-linear workload
    (1, 1024, 4096, 3, 6.0, False),     # one token, the longest row the kernel takes
    (5, 300, 272, 4, 6.0, True),        # ragged N (a partial weight tile) and ragged K (a partial box)
    (16, 4096, 1024, 0, 6.0, True),     # 32 tiles, no outliers
    (9, 2048, 2064, 40, 6.0, False),    # many outlier columns spread over every stage
    (12, 512, 1024, 3, 0.0, True),      # threshold 0
    (4, 16384, 512, 2, 6.0, True),      # 128 tiles: one CTA per tile (no K split)
    (7, 2048, 1152, 9, 6.0, True),      # 9 boxes over a cluster of 8: one CTA takes two
]


@pytest.mark.parametrize("M,N,K,n_out,tau,with_bias", SMALL_SHAPES)
def test_small_forward_against_oracle_and_two_stage(i8, M, N, K, n_out, tau, with_bias):
    """For few tokens and a small weight the forward is one kernel; the two-stage path
    (i8_linear8bit_prepare + i8_linear8bit_matmul_dequant) computes the same values with
    other kernels.  Both are checked against the oracle, and against each other."""
    X, _ = act(M, K, n_out, mag=(8.0, 60.0), seed=31 + M)
    W = wl.weight(32 + N, N, K)
    b = wl.bias(33, N) if with_bias else None
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    dX, dCB, dSCB, db = dev(X), dev(rCB), dev(rSCB), None if b is None else dev(b)
    out, ws = i8.i8_linear8bit_forward(dX, dCB, dSCB, db, tau)
    code, count = i8.i8_read_status(ws)
    _, _, cols = oracle.quantize_rowwise(X, tau)
    assert code == 0 and count == (len(cols) if tau > 0 else 0)
    ref = oracle.linear8bit_forward(X, rCB, rSCB, b, tau)
    assert_close(host(out), ref, "one-launch forward")
    two = torch.empty_like(out)
    i8.i8_linear8bit_prepare(dX, dCB, tau, ws, 256)
    i8.i8_linear8bit_matmul_dequant(dCB, dSCB, db, M, tau, two, ws, 256)
    assert i8.i8_read_status(ws) == (code, count)
    assert_close(host(two), ref, "two-stage forward")
    assert_close(host(out), host(two).astype(np.float64), "one-launch vs two-stage")


def test_small_forward_repeat_is_deterministic(i8):
    X, _ = act(16, 1024, 2, seed=40)
    W = wl.weight(41, 1024, 1024)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    dX, dCB, dSCB = dev(X), dev(rCB), dev(rSCB)
    a, ws = i8.i8_linear8bit_forward(dX, dCB, dSCB, None, 6.0)
    for _ in range(3):
        b, _ = i8.i8_linear8bit_forward(dX, dCB, dSCB, None, 6.0, workspace=ws)
        assert torch.equal(a, b)


# ------------------------------------------------------------------ CUDA graph capture
@pytest.mark.parametrize("M,N,K,n_out", [(256, 512, 1024, 3), (4, 4096, 8192, 5), (16, 1024, 1024, 2)])
def test_forward_cuda_graph_replay(i8, M, N, K, n_out):
    """The forward never waits for the host: it can be captured once and replayed on new
    inputs (a different outlier set each time), the outlier columns being found on the device."""
    X1, _ = act(M, K, n_out, seed=21)
    X2, _ = act(M, K, n_out + 2, seed=22)
    W = wl.weight(23, N, K)
    b = wl.bias(24, N)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    dX, dCB, dSCB, db = dev(X1), dev(rCB), dev(rSCB), dev(b)
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws = torch.empty((i8.i8_linear8bit_workspace_size(M, N, K, 256),), dtype=torch.uint8, device="cuda")
    i8.i8_linear8bit_forward(dX, dCB, dSCB, db, 6.0, out=out, workspace=ws)  # first call outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        i8.i8_linear8bit_forward(dX, dCB, dSCB, db, 6.0, out=out, workspace=ws)
    for X in (X2, X1):
        dX.copy_(torch.from_numpy(X).cuda())
        graph.replay()
        torch.cuda.synchronize()
        _, _, cols = oracle.quantize_rowwise(X, 6.0)
        assert i8.i8_read_status(ws) == (0, len(cols))
        assert_close(host(out), oracle.linear8bit_forward(X, rCB, rSCB, b, 6.0), "graph replay")


# ------------------------------------------------------------------ input gradient
@pytest.mark.parametrize("N,K", [(8, 16), (200, 48), (1000, 2064), (4096, 4096), (11008, 4096), (4096, 11008)])
def test_dequant_transposed_bit_exact(i8, N, K):
    """Wt = dequant(CB, SCB)^T bit for bit (the fp32 two-step evaluation equals the oracle's
    single rounding for every code and scale, so no tolerance is needed)."""
    W = wl.weight(N * 3 + K, N, K)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    dCB, dSCB = dev(rCB), dev(rSCB)
    Wt = host(i8.i8_dequant_transposed(dCB, dSCB))
    ref = np.ascontiguousarray(oracle.dequant(rCB, rSCB).T)
    assert Wt.shape == (K, N)
    assert np.array_equal(Wt.view(np.uint16), ref.view(np.uint16))
    assert np.array_equal(Wt.T, host(i8.i8_dequant(dCB, dSCB)))


def assert_grad_close(got, ref, dY, W_hat, what=""):
    """|gpu - oracle| <= n * 2^-23 * sum_n |dY[i, n] W^[n, k]| + ulp16: fp32 accumulation of
    exact fp16 x fp16 products in any order (a per-add error of at most 2^-23, allowing
    truncating adds), then one fp16 rounding on each side."""
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape
    n = dY.shape[1]
    S = np.abs(dY.astype(np.float64)) @ np.abs(W_hat.astype(np.float64))
    ulp = np.spacing(np.maximum(np.abs(g), np.abs(r)).astype(np.float16)).astype(np.float64)
    bound = n * 2.0 ** -23 * S + ulp
    d = np.abs(g - r)
    bad = d > bound
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} out of bound; first {i} got {g[i]} "
                             f"want {r[i]} bound {bound[i]:.3g}; max abs {d.max():.3g}")


BSHAPES = [(1, 8, 16), (130, 72, 48), (512, 1024, 768), (1024, 4096, 4096), (2048, 4096, 4096),
           (300, 4104, 528), (4096, 4096, 11008)]


@pytest.mark.parametrize("M,N,K", BSHAPES)
def test_backward_input(i8, M, N, K):
    """dX = dY . dequant(CB, SCB) through the tcgen05 fp16 GEMM, against the oracle."""
    dY = wl.grad_output(M + 2 * N + 3 * K, M, N)
    W = wl.weight(M + N + K, N, K)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    Wt = i8.i8_dequant_transposed(dev(rCB), dev(rSCB))
    dX = host(i8.i8_linear8bit_backward_input(dev(dY), Wt))
    rows = None if M <= 2048 else np.random.default_rng(M).choice(M, 256, replace=False)
    ref = oracle.linear8bit_backward_input(dY, rCB, rSCB, rows=rows)
    sel = dY if rows is None else dY[rows]
    assert_grad_close(dX if rows is None else dX[rows], ref, sel, oracle.dequant(rCB, rSCB), "backward_input")


def test_backward_input_plain_store_edge(i8):
    """An output width that is not a multiple of 8 takes the plain-store epilogue."""
    M, N, K = 100, 64, 20
    dY = wl.grad_output(7, M, N)
    rCB, rSCB = oracle.quantize_weight_rowwise(wl.weight(8, N, K))
    W_hat = oracle.dequant(rCB, rSCB)
    dX = host(i8.i8_linear8bit_backward_input(dev(dY), dev(np.ascontiguousarray(W_hat.T))))
    assert_grad_close(dX, oracle.linear8bit_backward_input(dY, rCB, rSCB), dY, W_hat, "plain store")


def test_backward_input_repeat_is_deterministic(i8):
    dY = dev(wl.grad_output(9, 640, 2048))
    rCB, rSCB = oracle.quantize_weight_rowwise(wl.weight(10, 2048, 1536))
    Wt = i8.i8_dequant_transposed(dev(rCB), dev(rSCB))
    a = host(i8.i8_linear8bit_backward_input(dY, Wt))
    b = host(i8.i8_linear8bit_backward_input(dY, Wt))
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


# ------------------------------------------------------------------ several weights, one X
MSHAPES = [
    (300, 1040, (520, 264, 1040), 3, 6.0),    # prefill, few outlier columns
    (512, 1024, (4096, 4096), 40, 6.0),       # prefill, > 16 columns: tcgen05 fp16 outlier path
    (300, 1040, (520, 264), 3, 0.0),          # threshold 0
    (7, 2064, (1000, 272, 4096), 5, 6.0),     # few tokens: two one-launch weights, one decode GEMM
    (16, 4096, (4096, 1024), 40, 6.0),        # few tokens, many outlier columns (one of each path)
    (5, 1024, (1024, 512, 264), 3, 6.0),      # few tokens, every weight one-launch
]


@pytest.mark.parametrize("M,K,Ns,n_out,tau", MSHAPES)
def test_forward_multi_matches_single(i8, M, K, Ns, n_out, tau):
    """Each output of the multi-weight forward is bit for bit the single forward of that
    weight (same X), and within tolerance of the oracle."""
    X, _ = act(M, K, n_out, seed=M + K + len(Ns))
    dXd = dev(X)
    ws_ref, CBs, SCBs, biases, host_w = [], [], [], [], []
    for g, N in enumerate(Ns):
        W = wl.weight(40 + g, N, K)
        CB, SCB, _ = i8.i8_quantize_rowwise(dev(W), 0.0)
        b = wl.bias(50 + g, N) if g % 2 == 0 else None
        CBs.append(CB)
        SCBs.append(SCB)
        biases.append(None if b is None else dev(b))
        host_w.append((W, b))
    outs, ws = i8.i8_linear8bit_forward_multi(dXd, CBs, SCBs, biases, tau)
    code, count = i8.i8_read_status(ws)
    _, _, rcols = oracle.quantize_rowwise(X, tau)
    assert code == 0
    assert count == (len(rcols) if tau > 0 else 0)
    for g in range(len(Ns)):
        single, _ = i8.i8_linear8bit_forward(dXd, CBs[g], SCBs[g], biases[g], tau)
        got = host(outs[g])
        assert np.array_equal(got.view(np.uint16), host(single).view(np.uint16)), g
        rCB, rSCB = oracle.quantize_weight_rowwise(host_w[g][0])
        assert_close(got, oracle.linear8bit_forward(X, rCB, rSCB, host_w[g][1], tau), f"multi weight {g}")


def test_forward_multi_reuses_workspace(i8):
    """A second call on the same workspace with a different X (another outlier set) is correct:
    the per-call state (status, counts, bitmap, split-K counters) is rebuilt each time."""
    for M in (300, 9):
        K, Ns = 1024, (768, 256)
        W = [wl.weight(60 + g, N, K) for g, N in enumerate(Ns)]
        CBs, SCBs = zip(*[i8.i8_quantize_rowwise(dev(w), 0.0)[:2] for w in W])
        ws = torch.empty((i8.i8_linear8bit_multi_workspace_size(M, K, list(Ns), 256),), dtype=torch.uint8,
                         device="cuda")
        for seed, n_out in ((70, 6), (71, 2)):
            X, _ = act(M, K, n_out, seed=seed)
            outs, _ = i8.i8_linear8bit_forward_multi(dev(X), list(CBs), list(SCBs), None, 6.0, workspace=ws)
            code, count = i8.i8_read_status(ws)
            _, _, rcols = oracle.quantize_rowwise(X, 6.0)
            assert (code, count) == (0, len(rcols))
            for g in range(len(Ns)):
                rCB, rSCB = oracle.quantize_weight_rowwise(W[g])
                assert_close(host(outs[g]), oracle.linear8bit_forward(X, rCB, rSCB, None, 6.0), f"reuse {M} {g}")


@pytest.mark.parametrize("M,N,K", [(16, 1024, 1024), (3, 300, 272), (300, 520, 1040)])
def test_layer_matches_function(i8, M, N, K):
    """Linear8bitLt (weights checked once, a workspace per token count) gives the function's
    output bit for bit, call after call, and the oracle's within tolerance."""
    X, _ = act(M, K, 3, mag=(8.0, 60.0), seed=61 + M)
    W = wl.weight(62 + N, N, K)
    b = wl.bias(63, N)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    dCB, dSCB, db = dev(rCB), dev(rSCB), dev(b)
    layer = i8.Linear8bitLt(dCB, dSCB, db, 6.0)
    ref_out, ws = i8.i8_linear8bit_forward(dev(X), dCB, dSCB, db, 6.0)
    for _ in range(2):
        o = layer(dev(X))
        assert torch.equal(o, ref_out)
        assert i8.i8_read_status(layer.last_workspace) == i8.i8_read_status(ws)
    assert_close(host(o), oracle.linear8bit_forward(X, rCB, rSCB, b, 6.0), "layer")
