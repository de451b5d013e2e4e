"""GPU checks of the column-parallel split (the host logic with two ranks is in
test_multirank.py, on CPU):

* i8_gather_column_blocks puts rank-major blocks in place, bit for bit;
* each rank's forward on its rows of the weight matches the oracle's columns of
  the whole layer, and the reordered blocks match the whole output (the ranks
  are run one after another on the one GPU: they do not wait on each other);
* the split class at world size 1 is the plain forward.
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
    g, r = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    bad = np.abs(g - r) > ATOL + RTOL * np.abs(r)
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} out of tolerance, max abs {np.abs(g - r).max():.3g}"


@pytest.mark.parametrize("P,M,Np", [(2, 300, 520), (4, 7, 13), (8, 4096, 512), (1, 16, 24)])
def test_gather_column_blocks_bit_exact(i8, P, M, Np):
    G = np.random.default_rng(P * M + Np).standard_normal((P, M, Np)).astype(np.float16)
    out = host(i8.i8_gather_column_blocks(dev(G)))
    want = np.transpose(G, (1, 0, 2)).reshape(M, P * Np)
    assert np.array_equal(out.view(np.uint16), want.view(np.uint16))


@pytest.mark.parametrize("M,N,K,n_out,P", [(512, 4096, 1024, 4, 2), (16, 4096, 4096, 8, 4), (2048, 13824, 5120, 51, 2)])
def test_shards_match_oracle_columns(i8, M, N, K, n_out, P):
    from int8_mixed_precision_vectorwise_b200 import column_parallel as cp
    X, _ = wl.activation(wl.BASE_SEED + 800 + M, M, K, n_out, (6.0, 80.0))
    W = wl.weight(801, N, K)
    b = wl.bias(802, N)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    rows = np.arange(M) if M <= 256 else np.random.default_rng(M).choice(M, 256, replace=False)
    ref = oracle.linear8bit_forward(X, rCB, rSCB, b, 6.0, rows=rows)
    dX = dev(X)
    blocks = []
    for p in range(P):
        n0, n1 = cp.shard_range(N, P, p)
        out_p, ws = i8.i8_linear8bit_forward(dX, dev(rCB[n0:n1]), dev(rSCB[n0:n1]), dev(b[n0:n1]), 6.0)
        code, count = i8.i8_read_status(ws)
        assert code == 0
        assert_close(host(out_p)[rows], ref[:, n0:n1], f"shard {p}")
        blocks.append(out_p)
    out = host(i8.i8_gather_column_blocks(torch.stack(blocks)))
    assert_close(out[rows], ref, "gathered")


def test_world_one_is_the_plain_forward(i8):
    from int8_mixed_precision_vectorwise_b200 import column_parallel as cp
    M, N, K = 300, 1024, 2048
    X, _ = wl.activation(wl.BASE_SEED + 810, M, K, 3, (20.0, 60.0))
    CB, SCB, _ = i8.i8_quantize_rowwise(dev(wl.weight(811, N, K)), 0.0)
    b = dev(wl.bias(812, N))
    layer = cp.ColumnParallelLinear8bit(CB, SCB, b, threshold=6.0)
    got = layer(dev(X))
    assert layer.status()[0] == 0
    want, _ = i8.i8_linear8bit_forward(dev(X), CB, SCB, b, 6.0)
    assert torch.equal(got, want)
