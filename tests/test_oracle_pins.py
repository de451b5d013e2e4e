"""Pins for the CPU oracle against facts fixed by the pages and by mathematics.

None of these re-types the oracle's formulas: they use hand-derived closed-form
cases (tests/golden/closed_form_cases.json), error bounds of row-wise absmax
rounding, algebraic invariants, brute force with Python integers, and special
cases that reduce to textbook formulas (threshold 0 -> plain int8 dequant; all
columns outliers -> an fp16-path matmul against the dequantised weight).
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")))


def f16(a):
    return np.asarray(a, dtype=np.float16)


# ---------------------------------------------------------------- closed form
@pytest.mark.parametrize("case", GOLD["quantize"], ids=lambda c: c["name"])
def test_quantize_closed_form(case):
    CA, SCA, cols = oracle.quantize_rowwise(f16(case["X"]), case["threshold"])
    assert CA.tolist() == case["CA"]
    assert SCA.tolist() == [float(np.float32(v)) for v in case["SCA"]]
    assert cols.tolist() == case["cols"]


@pytest.mark.parametrize("case", GOLD["matmul"], ids=lambda c: c["name"])
def test_matmul_closed_form(case):
    C = oracle.int8_linear_matmul(np.array(case["A"], np.int8), np.array(case["B"], np.int8))
    assert C.dtype == np.int32
    assert C.tolist() == case["C"]


@pytest.mark.parametrize("case", GOLD["mm_dequant"], ids=lambda c: c["name"])
def test_mm_dequant_closed_form(case):
    b = None if case["bias"] is None else f16(case["bias"])
    out = oracle.int8_mm_dequant(np.array(case["C"], np.int32), np.float32(case["SCA"]),
                                 np.float32(case["SCB"]), b)
    assert out.dtype == np.float16
    assert out.astype(np.float64).tolist() == case["out"]


@pytest.mark.parametrize("case", GOLD["dequant"], ids=lambda c: c["name"])
def test_dequant_closed_form(case):
    W = oracle.dequant(np.array(case["CB"], np.int8), np.float32(case["SCB"]))
    assert W.astype(np.float64).tolist() == case["W"]


@pytest.mark.parametrize("case", GOLD["backward"], ids=lambda c: c["name"])
def test_backward_input_closed_form(case):
    dX = oracle.linear8bit_backward_input(f16(case["dY"]), np.array(case["CB"], np.int8), np.float32(case["SCB"]))
    assert dX.dtype == np.float16
    assert dX.tolist() == case["dX"]


@pytest.mark.parametrize("case", GOLD["forward"], ids=lambda c: c["name"])
def test_forward_closed_form(case):
    out = oracle.linear8bit_forward(f16(case["X"]), np.array(case["CB"], np.int8),
                                    np.float32(case["SCB"]), f16(case["bias"]), case["threshold"])
    assert out.astype(np.float64).tolist() == case["out"]


# ---------------------------------------------------------------- error bound
def _quant_error_ok(X, tau):
    CA, SCA, cols = oracle.quantize_rowwise(X, tau)
    x = X.astype(np.float64)
    keep = np.ones(X.shape[1], bool)
    keep[cols] = False
    s = SCA.astype(np.float64)[:, None]
    err = np.abs(x - CA.astype(np.float64) * s / 127.0)[:, keep]
    bound = (s / 254.0) * (1 + 2.0 ** -20) + 0.0
    # elements at or above the threshold in non-outlier columns cannot exist
    return bool(np.all(err <= np.broadcast_to(bound, (X.shape[0], X.shape[1]))[:, keep]))


@pytest.mark.parametrize("seed,M,K,tau", [(0, 7, 33, 0.0), (1, 16, 64, 6.0), (2, 64, 256, 2.5),
                                          (3, 5, 1024, 0.0), (4, 128, 96, 1.0)])
def test_quant_error_bound(seed, M, K, tau):
    """|x - CA*SCA/127| <= SCA/254 (plus fp32 slack) on every int8-path element."""
    g = np.random.default_rng(seed)
    X = (g.standard_normal((M, K)) * g.uniform(0.1, 4, size=(M, 1))).astype(np.float16)
    X[:, :3] *= 8  # some outliers when tau > 0
    assert _quant_error_ok(X, tau)


def test_row_max_maps_to_127():
    """The row's largest kept magnitude is coded +-127: SCA is the absmax, not another statistic."""
    g = np.random.default_rng(7)
    X = g.standard_normal((50, 40)).astype(np.float16)
    CA, SCA, cols = oracle.quantize_rowwise(X, 0.0)
    assert cols.size == 0
    assert np.all(np.abs(CA).max(axis=1) == 127)
    assert np.array_equal(SCA, np.abs(X.astype(np.float32)).max(axis=1))


# ---------------------------------------------------------------- brute force
def _brute_codes_row(row, tau):
    """Python-integer brute force for one row, with the fp32 rounding modelled by
    exhaustive search: the code is the integer nearest to fl32(x*fl32(127/s))."""
    vals = [float(v) for v in row]
    kept = [abs(v) for v in vals if tau == 0 or abs(v) < tau]
    s = max(kept) if kept else 0.0
    out = []
    for v in vals:
        if s == 0.0:
            out.append(0)
            continue
        p = Fraction(float(np.float32(v) * (np.float32(127.0) / np.float32(s))))
        # nearest integer, ties to even, by exhaustive comparison over -128..128
        best = None
        for q in range(-130, 131):
            d = abs(p - q)
            if best is None or d < best[0] or (d == best[0] and q % 2 == 0):
                best = (d, q)
        out.append(max(-127, min(127, best[1])))
    return s, out


def test_brute_force_grid():
    """Every 1x3 row over a grid that includes exact threshold hits and near misses."""
    grid = [0.0, 0.5, -0.5, 1.0, -3.0, 5.99609375, -5.99609375, 6.0, -6.0, 7.0, 0.00048828125]
    tau = 6.0
    rows = [[a, b, c] for a in grid for b in grid for c in grid]
    X = f16(rows)
    CA, SCA, cols = oracle.quantize_rowwise(X, tau)
    # column set: any element at or above the threshold
    want_cols = sorted({j for r in rows for j, v in enumerate(r) if abs(v) >= tau})
    assert cols.tolist() == want_cols
    for i, r in enumerate(rows):
        s, codes = _brute_codes_row(r, tau)
        assert float(SCA[i]) == s
        for j in range(3):
            want = 0 if j in want_cols else codes[j]
            assert int(CA[i, j]) == want, (r, j)


def test_brute_force_per_row_with_local_outliers():
    """Tiny random matrices, brute-forced row by row (threshold 2.0)."""
    g = np.random.default_rng(11)
    for _ in range(20):
        M, K = g.integers(1, 6), g.integers(1, 9)
        X = (g.standard_normal((M, K)) * 1.5).astype(np.float16)
        CA, SCA, cols = oracle.quantize_rowwise(X, 2.0)
        want_cols = sorted({j for i in range(M) for j in range(K) if abs(float(X[i, j])) >= 2.0})
        assert cols.tolist() == want_cols
        for i in range(M):
            s, codes = _brute_codes_row(X[i], 2.0)
            assert float(SCA[i]) == s
            for j in range(K):
                assert int(CA[i, j]) == (0 if j in want_cols else codes[j])


def test_matmul_brute_force():
    g = np.random.default_rng(3)
    for M, N, K in [(1, 1, 1), (3, 5, 7), (8, 4, 33), (2, 9, 128)]:
        A = g.integers(-128, 128, size=(M, K), dtype=np.int8)
        B = g.integers(-128, 128, size=(N, K), dtype=np.int8)
        C = oracle.int8_linear_matmul(A, B)
        for i in range(M):
            for n in range(N):
                assert int(C[i, n]) == sum(int(A[i, k]) * int(B[n, k]) for k in range(K))


def test_matmul_int64_library_agrees_large():
    """Exactness of the float64 product versus numpy's integer matmul at the largest K."""
    g = np.random.default_rng(5)
    A = g.integers(-127, 128, size=(3, 28672), dtype=np.int8)
    B = g.integers(-127, 128, size=(4, 28672), dtype=np.int8)
    A[0] = 127
    B[0] = 127
    C = oracle.int8_linear_matmul(A, B)
    ref = A.astype(np.int64) @ B.astype(np.int64).T
    assert np.array_equal(C.astype(np.int64), ref)
    assert int(C[0, 0]) == 16129 * 28672


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("p", [-3, 2, 5])
def test_power_of_two_scaling(p):
    g = np.random.default_rng(9)
    X = g.standard_normal((20, 64)).astype(np.float16)
    X[:, 5] = 9.0
    tau = 6.0
    CA, SCA, cols = oracle.quantize_rowwise(X, tau)
    Xs = (X.astype(np.float32) * 2.0 ** p).astype(np.float16)
    assert np.array_equal(Xs.astype(np.float32), X.astype(np.float32) * 2.0 ** p)  # exact in fp16
    CA2, SCA2, cols2 = oracle.quantize_rowwise(Xs, tau * 2.0 ** p)
    assert np.array_equal(CA, CA2)
    assert np.array_equal(cols, cols2)
    assert np.array_equal(SCA2, SCA * np.float32(2.0 ** p))


def test_sign_symmetry():
    g = np.random.default_rng(10)
    X = g.standard_normal((30, 48)).astype(np.float16)
    X[:, 7] = -7.0
    CA, SCA, cols = oracle.quantize_rowwise(X, 6.0)
    CAn, SCAn, colsn = oracle.quantize_rowwise(-X, 6.0)
    assert np.array_equal(CAn, -CA)
    assert np.array_equal(SCA, SCAn)
    assert np.array_equal(cols, colsn)


def test_column_permutation_equivariance():
    g = np.random.default_rng(12)
    X = g.standard_normal((16, 40)).astype(np.float16)
    X[:, [3, 30]] = 12.0
    perm = g.permutation(40)
    CA, SCA, cols = oracle.quantize_rowwise(X, 6.0)
    CAp, SCAp, colsp = oracle.quantize_rowwise(X[:, perm], 6.0)
    assert np.array_equal(CAp, CA[:, perm])
    assert np.array_equal(SCAp, SCA)
    assert sorted(perm[colsp].tolist()) == cols.tolist()   # new column p is old column perm[p]


def test_outlier_set_is_union_over_rows():
    """A big value in one row makes the whole column fp16 for every row."""
    X = f16([[1, 2, 3], [1, 2, 9], [1, 2, 3]])
    CA, SCA, cols = oracle.quantize_rowwise(X, 6.0)
    assert cols.tolist() == [2]
    assert np.all(CA[:, 2] == 0)
    assert SCA.tolist() == [3.0, 2.0, 3.0]


def test_bitmap_layout():
    words = oracle.outlier_bitmap([0, 31, 32, 70], 100)
    assert words.tolist() == [0x80000001, 0x1, 0x40, 0x0]


# ---------------------------------------------------------------- special cases
def _case(seed, M, K, N, n_out, mag=(20, 60), with_bias=True):
    g = np.random.default_rng(seed)
    X = g.standard_normal((M, K)).astype(np.float32)
    cols = np.sort(g.permutation(K)[:n_out])
    X[:, cols] = np.sign(g.standard_normal((M, n_out))) * g.uniform(*mag, size=(M, n_out))
    X = X.astype(np.float16)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float16)
    CB, SCB = oracle.quantize_weight_rowwise(W)
    b = (g.standard_normal(N) * 0.01).astype(np.float16) if with_bias else None
    return X, W, CB, SCB, b


def test_threshold_zero_is_plain_int8():
    """threshold 0: out == textbook row/col-scaled int8 product + bias (no fp16 part)."""
    X, W, CB, SCB, b = _case(20, 12, 96, 10, 2)
    out = oracle.linear8bit_forward(X, CB, SCB, b, 0.0)
    # textbook: quantise rows by absmax, integer product, outer-product rescale
    x = X.astype(np.float64)
    s = np.abs(x).max(axis=1)
    q = np.array([[int(np.rint(np.float32(v) * (np.float32(127) / np.float32(si)))) for v in row]
                  for row, si in zip(x, s)], dtype=np.int64)
    C = q @ CB.astype(np.int64).T
    y = C * s[:, None] * SCB.astype(np.float64)[None, :] / 16129.0 + b.astype(np.float64)
    assert np.array_equal(out, y.astype(np.float16))


def test_all_columns_outliers_is_fp16_matmul():
    """Every column an outlier: CA == 0 and out == X . (CB*SCB/127)^T + bias."""
    X, W, CB, SCB, b = _case(21, 9, 64, 11, 0)
    tau = 1e-3
    X[0] = np.where(np.abs(X[0]) < 1e-2, np.float16(0.5), X[0])   # every column hits tau in row 0
    CA, SCA, cols = oracle.quantize_rowwise(X, tau)
    assert cols.size == X.shape[1] and not CA.any()
    out = oracle.linear8bit_forward(X, CB, SCB, b, tau)
    Wdq = CB.astype(np.float64) * SCB.astype(np.float64)[:, None] / 127.0
    ref = X.astype(np.float64) @ Wdq.T + b.astype(np.float64)
    np.testing.assert_array_equal(out, ref.astype(np.float16))


def test_exact_grid_decomposition():
    """Rows on the exact grid k*SCA/127 have no quantisation error, so the mixed
    decomposition must equal X . Wdq^T + bias (no double counting, no dropped
    outlier term, correct 127 and 127^2 factors)."""
    g = np.random.default_rng(22)
    M, K, N = 6, 40, 7
    k = g.integers(-127, 128, size=(M, K))
    X = (k / 32.0).astype(np.float16)            # SCA grid 127/32, r = 32
    X[:, 0] = 127 / 32.0
    X[:, [5, 17]] = np.float16(23.5)             # outlier columns
    X[2, 17] = np.float16(-0.25)                 # small value inside an outlier column
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float16)
    CB, SCB = oracle.quantize_weight_rowwise(W)
    b = (g.standard_normal(N) * 0.01).astype(np.float16)
    out = oracle.linear8bit_forward(X, CB, SCB, b, 6.0)
    Wdq = CB.astype(np.float64) * SCB.astype(np.float64)[:, None] / 127.0
    ref = X.astype(np.float64) @ Wdq.T + b.astype(np.float64)
    np.testing.assert_array_equal(out, ref.astype(np.float16))


def test_forward_close_to_fp16_weights():
    """Informational bound vs the unquantised weight: error <= activation rounding
    + weight rounding bounds (per-element half steps), summed over K."""
    X, W, CB, SCB, b = _case(23, 8, 128, 16, 1)
    out = oracle.linear8bit_forward(X, CB, SCB, b, 6.0).astype(np.float64)
    ref = X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)
    _, SCA, _ = oracle.quantize_rowwise(X, 6.0)
    bound = (np.abs(X.astype(np.float64)).sum(1)[:, None] * (SCB.astype(np.float64)[None, :] / 254)
             + SCA.astype(np.float64)[:, None] / 254 * np.abs(W.astype(np.float64)).sum(1)[None, :]) * 1.01 + 1e-2
    assert np.all(np.abs(out - ref) <= bound)


def test_row_subset_matches_full():
    X, W, CB, SCB, b = _case(24, 40, 64, 8, 3)
    full = oracle.linear8bit_forward(X, CB, SCB, b, 6.0)
    rows = [0, 7, 39]
    sub = oracle.linear8bit_forward(X, CB, SCB, b, 6.0, rows=rows)
    assert np.array_equal(sub, full[rows])


def test_weight_quant_is_threshold_zero():
    W = f16([[0.5, -0.25, 8.0], [0, 0, 0]])
    CB, SCB = oracle.quantize_weight_rowwise(W)
    assert CB.tolist() == [[8, -4, 127], [0, 0, 0]]   # r = 127/8 = 15.875: 7.9375 -> 8, -3.96875 -> -4
    assert SCB.tolist() == [8.0, 0.0]


# ---------------------------------------------------------------- input gradient
def _frozen_layer(seed, M, N, K):
    rng = np.random.default_rng(seed)
    W = f16(rng.normal(0.0, 0.02, (N, K)))
    CB, SCB = oracle.quantize_weight_rowwise(W)
    dY = f16(rng.normal(0.0, 1.0, (M, N)))
    return CB, SCB, dY


@pytest.mark.parametrize("seed,M,N,K", [(0, 5, 24, 40), (1, 33, 64, 16), (2, 8, 17, 48)])
def test_backward_input_is_autograd_gradient(seed, M, N, K):
    """The oracle's dX equals what torch autograd derives for y = X . W^T + b in float64
    (a transposed or mis-indexed product fails on these non-square shapes)."""
    import torch
    CB, SCB, dY = _frozen_layer(seed, M, N, K)
    W = torch.from_numpy(oracle.dequant(CB, SCB).astype(np.float64))
    X = torch.zeros((M, K), dtype=torch.float64, requires_grad=True)
    b = torch.ones(N, dtype=torch.float64)
    y = X @ W.T + b
    (y * torch.from_numpy(dY.astype(np.float64))).sum().backward()
    got = oracle.linear8bit_backward_input(dY, CB, SCB)
    assert got.shape == (M, K)
    assert np.array_equal(got, X.grad.numpy().astype(np.float16))


def test_backward_input_one_hot_rows_select_weight_rows():
    """dY = e_n picks row n of the dequantised weight, exactly."""
    CB, SCB, _ = _frozen_layer(3, 1, 12, 32)
    dY = f16(np.eye(12))
    assert np.array_equal(oracle.linear8bit_backward_input(dY, CB, SCB), oracle.dequant(CB, SCB))


def test_backward_input_brute_force():
    """Exact rational sums with Python integers / fractions on a tiny case."""
    CB, SCB, dY = _frozen_layer(4, 3, 5, 4)
    W = oracle.dequant(CB, SCB)
    got = oracle.linear8bit_backward_input(dY, CB, SCB)
    for i in range(3):
        for k in range(4):
            s = sum(Fraction(float(dY[i, n])) * Fraction(float(W[n, k])) for n in range(5))
            assert got[i, k] == np.float16(float(s))


def test_backward_input_row_subset():
    CB, SCB, dY = _frozen_layer(5, 9, 16, 32)
    full = oracle.linear8bit_backward_input(dY, CB, SCB)
    assert np.array_equal(oracle.linear8bit_backward_input(dY, CB, SCB, rows=[8, 0, 3]), full[[8, 0, 3]])


def test_dequant_two_step_fp32_equals_one_rounding():
    """For every code c in [-127, 127] and every positive finite fp16 row scale, evaluating
    fp16(fl32(c * fl32(SCB / 127))) gives the oracle's once-rounded fp16(c * SCB / 127):
    the exact value c * SCB / 127 never lies within 2^-18 (relative) of an fp16 rounding
    boundary unless it is on one, and then it is representable.  So a GPU dequantiser that
    takes those two fp32 steps can be compared with the oracle bit for bit."""
    scb = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    s = scb / np.float32(127.0)
    for c in range(-127, 128):
        two = (np.float32(c) * s).astype(np.float16)
        one = oracle.dequant(np.full((scb.size, 1), c, np.int8), scb)[:, 0]
        assert np.array_equal(two.view(np.uint16), one.view(np.uint16)), c
