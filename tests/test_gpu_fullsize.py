"""Full-size parity on the five workload families, in the launch configuration
bench.py times (i8_linear8bit_forward with the same max_outlier_cols).

Codes, absmax scales and outlier bitmaps are compared in full (bit-exact);
int32 accumulators and fp16 outputs on all rows when a layer has at most 256,
else on a seeded sample of at least 256 rows (times every output column) that
also spans the first/last tiles and the ragged edge (the oracle evaluates
exactly those rows; its outlier set is still the union over every row).  For
16 tokens or fewer the int32 sums are also taken from the few-token stream-K
kernel the forward uses (i8_int8_linear_matmul_ws) and compared in full.
"""

import numpy as np
import pytest
import torch

import oracle
from int8_mixed_precision_vectorwise_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 1e-3
MAX_OUTLIER_COLS = 256   # as in bench.py


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


def sample_rows(M, n=256, seed=0):
    """All rows if M <= n, else n distinct seeded rows plus the tile edges."""
    if M <= n:
        return np.arange(M, dtype=np.int64)
    g = np.random.default_rng(seed)
    fixed = {0, 1, 127, 128, 255, 256, M // 2, M - 1, max(M - 128, 0), max(M - 129, 0)}
    extra = set(g.choice(M, size=n, replace=False).tolist())
    return np.array(sorted(r for r in fixed | extra if 0 <= r < M), dtype=np.int64)


def check_close(got, ref, what):
    g, r = got.astype(np.float64), ref.astype(np.float64)
    bad = np.abs(g - r) > ATOL + RTOL * np.abs(r)
    assert not bad.any(), f"{what}: {int(bad.sum())} out of tolerance, max abs {np.abs(g - r).max():.3g}"


_weight_cache = {}


def weights(i8, key, li, L):
    """(host W, oracle CB/SCB, device CB/SCB) with the GPU weight prep checked bit-exact."""
    k = (key, li)
    if k not in _weight_cache:
        _, _, W, b = wl.layer_inputs(wl.seed_of(key), li, L)
        rCB, rSCB = oracle.quantize_weight_rowwise(W)
        CB, SCB, _ = i8.i8_quantize_rowwise(dev(W), 0.0)
        assert np.array_equal(host(SCB).view(np.uint32), rSCB.view(np.uint32))
        assert np.array_equal(host(CB), rCB)
        _weight_cache.clear()
        _weight_cache[k] = (rCB, rSCB, CB, SCB, b)
    return _weight_cache[k]


def run_layer(i8, key, li, L, X):
    rCB, rSCB, CB, SCB, b = weights(i8, key, li, L)
    dX = dev(X)
    # quantiser: full bit-exact check
    CA, SCA, bm = i8.i8_quantize_rowwise(dX, L.threshold)
    rCA, rSCA, rcols = oracle.quantize_rowwise(X, L.threshold)
    assert np.array_equal(host(SCA).view(np.uint32), rSCA.view(np.uint32))
    assert np.array_equal(host(CA), rCA)
    if L.threshold > 0:
        assert np.array_equal(host(bm).view(np.uint32), oracle.outlier_bitmap(rcols, L.K))
    rows = sample_rows(L.M, seed=li)
    assert len(rows) >= min(L.M, 256)
    # int32 accumulators on the sampled rows (GPU GEMM over the full matrices)
    C = i8.i8_int8_linear_matmul(CA, CB)
    rC = oracle.int8_linear_matmul(rCA[rows], rCB)
    assert np.array_equal(host(C)[rows], rC)
    del C
    if L.M <= 16:
        # the few-token stream-K kernel's own int32 sums (split-K partials combined in its workspace)
        Cd, _ = i8.i8_int8_linear_matmul_ws(CA, CB)
        assert np.array_equal(host(Cd), rC)
        del Cd
    # fused forward, as bench.py launches it
    out, ws = i8.i8_linear8bit_forward(dX, CB, SCB, None if b is None else dev(b), L.threshold,
                                       max_outlier_cols=MAX_OUTLIER_COLS)
    code, count = i8.i8_read_status(ws)
    assert code == 0
    assert count == (len(rcols) if L.threshold > 0 else 0)
    ref = oracle.linear8bit_forward(X, rCB, rSCB, b, L.threshold, rows=rows)
    check_close(host(out)[rows], ref, f"{key}/{L.name}")


def layer_params(keys):
    W = wl.workloads()
    return [pytest.param(k, li, id=f"{k}-{L.name}") for k in keys for li, L in enumerate(W[k].layers)]


@pytest.mark.parametrize("key,li", layer_params(["C1"]))
def test_single_linear(i8, key, li):
    L = wl.workloads()[key].layers[li]
    X, _, _, _ = wl.layer_inputs(wl.seed_of(key), li, L)
    run_layer(i8, key, li, L, X)


# C3: the three distinct shapes (q/k/v/o share one, gate/up another)
@pytest.mark.parametrize("key,li", [pytest.param("C3", 0, id="C3-q_proj"), pytest.param("C3", 4, id="C3-gate_proj"),
                                    pytest.param("C3", 6, id="C3-down_proj")])
def test_llama7b_prefill(i8, key, li):
    L = wl.workloads()[key].layers[li]
    X, _, _, _ = wl.layer_inputs(wl.seed_of(key), li, L)
    run_layer(i8, key, li, L, X)


@pytest.mark.parametrize("key,li", layer_params(["C4_t1_o1", "C4_t16_o8", "C4_t4_o0", "C4_t4_o8", "C4_t16_o0"]))
def test_llama70b_decode(i8, key, li):
    L = wl.workloads()[key].layers[li]
    X, _, _, _ = wl.layer_inputs(wl.seed_of(key), li, L)
    run_layer(i8, key, li, L, X)


@pytest.mark.parametrize("key", ["C5_f0.0_t0", "C5_f0.001_t6", "C5_f0.01_t6", "C5_f0.05_t6", "C5_f0.05_t0"])
def test_llama13b_sweep(i8, key):
    L = wl.workloads()[key].layers[0]
    X, _, _, _ = wl.layer_inputs(wl.seed_of(key), 0, L)
    run_layer(i8, key, 0, L, X)
