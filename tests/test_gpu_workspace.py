"""GPU parity of what the forward computes before its fp16 output, read back
through the C ABI and compared with the CPU oracle bit for bit:

* the int32 sums of the few-token (stream-K) GEMM, through
  i8_int8_linear_matmul_ws, on shapes where a 128-row weight tile is split
  across several CTAs and where it is not;
* the prepared workspace of i8_linear8bit_prepare (codes with their outlier
  columns zeroed, row scales, the outlier list and counts, the bitmap, and the
  gathered fp16 operands X[:, O] and fp16(CB[:, O]) in their documented order),
  for the many-token and the few-token preparation;
* the status words of the gradient and raw-matmul entry points, and forwards
  running at once on two streams of one device.
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


def codes(seed, rows, cols):
    """Uniform int8 codes over the whole range the quantiser can emit, [-127, 127]."""
    return np.random.default_rng(seed).integers(-127, 128, size=(rows, cols), dtype=np.int64).astype(np.int8)


def assert_close(got, ref, what=""):
    g, r = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    bad = np.abs(g - r) > ATOL + RTOL * np.abs(r)
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} out of tolerance, max abs {np.abs(g - r).max():.3g}"


# ------------------------------------------------------------------ few-token GEMM, int32
def split_info(N, K, sms=148, stage_bytes=512, max_grid=256):
    """(grid, k-stages per CTA, most CTAs sharing one 128-row tile) of the stream-K split."""
    kb = -(-K // stage_bytes)
    total = -(-N // 128) * kb
    grid = min(sms, max_grid, total)
    per = -(-total // grid)
    most = max((((t + 1) * kb - 1) // per) - ((t * kb) // per) + 1 for t in range(-(-N // 128)))
    return grid, per, most


DECODE_SHAPES = [
    (1, 28672, 8192), (4, 28672, 8192), (16, 28672, 8192),     # Llama-70B FFN up / gate
    (1, 8192, 28672), (4, 8192, 28672), (16, 8192, 28672),     # Llama-70B FFN down
    (16, 1024, 512),     # every tile owned by one CTA (no split)
    (3, 1000, 1024),     # every tile split across 2 CTAs, ragged last tile
    (7, 300, 4112),      # 9 CTAs per tile, ragged K (not a multiple of the 512-byte stage)
    (16, 2000, 8192),    # 8 CTAs per tile
    (11, 16, 16),        # one tile, one partial stage
]


@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
def test_few_token_gemm_int32_bit_exact(i8, M, N, K):
    A = codes(100 + M, M, K)
    B = codes(200 + N, N, K)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    C, ws = i8.i8_int8_linear_matmul_ws(dev(A), dev(B), status=status)
    got = host(C)
    assert int(host(status)[0]) == 0
    assert np.array_equal(got, oracle.int8_linear_matmul(A, B))
    # a second call on the same workspace (its split-K counters start again from zero)
    C2, _ = i8.i8_int8_linear_matmul_ws(dev(A), dev(B), workspace=ws)
    assert np.array_equal(host(C2), got)


def test_few_token_split_cases_are_what_they_claim():
    """The shape list covers both sides of the split (checked on the host)."""
    assert split_info(1024, 512)[2] == 1
    assert split_info(1000, 1024)[2] == 2
    assert split_info(300, 4112)[2] == 9
    assert split_info(28672, 8192)[2] >= 2 and split_info(8192, 28672)[2] >= 3


def test_few_token_gemm_on_quantised_codes(i8):
    """The int32 sums the forward itself forms: CA from the quantiser (outlier columns zeroed)."""
    X, _ = wl.activation(wl.BASE_SEED + 77, 16, 8192, 8, (30.0, 30.0))
    W = wl.weight(78, 4096, 8192)
    rCA, _, _ = oracle.quantize_rowwise(X, 6.0)
    rCB, _ = oracle.quantize_weight_rowwise(W)
    C, _ = i8.i8_int8_linear_matmul_ws(dev(rCA), dev(rCB))
    assert np.array_equal(host(C), oracle.int8_linear_matmul(rCA, rCB))


def test_matmul_ws_many_rows_uses_tensor_core_gemm(i8):
    A, B = codes(5, 300, 1040), codes(6, 520, 1040)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    C, _ = i8.i8_int8_linear_matmul_ws(dev(A), dev(B), status=status)
    assert np.array_equal(host(C), oracle.int8_linear_matmul(A, B))
    assert int(host(status)[0]) == 0


# ------------------------------------------------------------------ prepared workspace
FRAG = [0, 1, 8, 9, 2, 3, 10, 11, 4, 5, 12, 13, 6, 7, 14, 15]   # entry held by each position of a group


def stored_entries(n_pos, many_tokens):
    """List entry held at each stored position of the gathered operands."""
    p = np.arange(n_pos)
    return 16 * (p // 16) + np.array(FRAG)[p % 16] if many_tokens else p


def ws_view(ws, off, dtype, count):
    nbytes = np.dtype(dtype).itemsize * count
    return host(ws[off:off + nbytes]).view(dtype)


PREP_CASES = [
    # M, N, K, planted outlier columns, threshold, capacity
    (300, 520, 1040, 5, 6.0, 64),      # <= 16 columns: one zero-padded group of 16
    (257, 384, 1024, 17, 6.0, 256),    # just past 16: zero padded to 64
    (130, 520, 1040, 70, 6.0, 256),    # two 64-column tiles
    (2048, 640, 5120, 250, 6.0, 256),  # ~5 % of the columns, near the capacity
    (200, 384, 512, 3, 0.0, 256),      # threshold 0: no list, nothing zeroed
    (16, 1024, 8192, 8, 6.0, 256),     # few tokens
    (1, 4096, 28672, 3, 6.0, 256),
    (4, 2048, 4096, 40, 6.0, 256),     # few tokens, outliers in every CTA's column range
    (16, 512, 28672, 40, 6.0, 256),    # few tokens on long rows: the 16-CTA preparation cluster
    (12, 256, 24576, 10, 6.0, 64),     # the same, 12 tokens, ragged column ranges
    (4, 256, 28672, 5, 6.0, 64),       # 4 tokens on long rows: also the 16-CTA cluster
    (300, 520, 1040, 80, 6.0, 101),    # 80 columns, a capacity that is not a multiple of 4
    (260, 300, 8192, 100, 6.0, 256),   # 100 columns on long rows
    # the preparation streams whole rows once there is a listed column per 48 bytes of row
    (300, 520, 8192, 40, 6.0, 256),    # 40 columns on 8192-byte rows: gathered, padded to 64
    (130, 264, 512, 12, 6.0, 256),     # 12 columns on 512-byte rows: streamed, one group of 16
    (70, 136, 1040, 33, 6.0, 40),      # streamed, ragged last chunk, capacity 40 < 64
]


@pytest.mark.parametrize("M,N,K,n_out,tau,cap", PREP_CASES)
def test_prepared_workspace_matches_oracle(i8, M, N, K, n_out, tau, cap):
    X, _ = wl.activation(wl.BASE_SEED + 300 + M, M, K, n_out, (6.0, 80.0))
    W = wl.weight(301 + N, N, K)
    rCB, _ = oracle.quantize_weight_rowwise(W)
    rCA, rSCA, cols = oracle.quantize_rowwise(X, tau)
    L = i8.i8_linear8bit_workspace_layout(M, N, K, cap)
    assert L["few_tokens"] == int(M <= 16)
    ws = torch.full((L["total"],), 0xA5, dtype=torch.uint8, device="cuda")   # stale bytes everywhere
    i8.i8_linear8bit_prepare(dev(X), dev(rCB), tau, ws, cap)
    total = len(cols)
    used = min(total, cap)
    hdr = ws_view(ws, L["header"], np.uint32, 3)
    assert hdr.tolist() == [0 if total <= cap else 6, used, total]
    assert np.array_equal(ws_view(ws, L["sca"], np.uint32, M), rSCA.view(np.uint32))
    assert np.array_equal(ws_view(ws, L["ca"], np.int8, M * K).reshape(M, K), rCA)
    if used == 0:
        return
    assert np.array_equal(ws_view(ws, L["idx"], np.int32, used), cols[:used])
    many = M > 16
    if many:
        assert np.array_equal(ws_view(ws, L["bitmap"], np.uint32, (K + 31) // 32), oracle.outlier_bitmap(cols, K))
    n_pos = (-(-used // 64) * 64 if used > 16 else 16) if many else -(-used // 16) * 16
    ent = stored_entries(n_pos, many)
    live = ent < used
    xo = ws_view(ws, L["x_o"], np.uint16, M * L["ld_o"]).reshape(M, L["ld_o"])[:, :n_pos]
    want = np.zeros((M, n_pos), np.uint16)
    want[:, live] = X[:, cols[ent[live]]].view(np.uint16)
    assert np.array_equal(xo, want), "gathered X[:, O]"
    if many:
        wo = ws_view(ws, L["w_o"], np.uint16, N * L["ld_o"]).reshape(N, L["ld_o"])[:, :n_pos]
        wwant = np.zeros((N, n_pos), np.uint16)
        wwant[:, live] = rCB[:, cols[ent[live]]].astype(np.float16).view(np.uint16)
        assert np.array_equal(wo, wwant), "gathered fp16(CB[:, O])"


@pytest.mark.parametrize("M", [64, 4])
def test_prepared_workspace_overflow(i8, M):
    """More outlier columns than the capacity: the status says so and the list holds the first ones."""
    N, K, cap = 256, 512, 8
    X, _ = wl.activation(wl.BASE_SEED + 400 + M, M, K, 20, (20.0, 60.0))
    rCB, _ = oracle.quantize_weight_rowwise(wl.weight(401, N, K))
    _, _, cols = oracle.quantize_rowwise(X, 6.0)
    L = i8.i8_linear8bit_workspace_layout(M, N, K, cap)
    ws = torch.zeros((L["total"],), dtype=torch.uint8, device="cuda")
    i8.i8_linear8bit_prepare(dev(X), dev(rCB), 6.0, ws, cap)
    assert ws_view(ws, L["header"], np.uint32, 3).tolist() == [6, cap, len(cols)]
    assert np.array_equal(ws_view(ws, L["idx"], np.int32, cap), cols[:cap])


# ------------------------------------------------------------------ status words, streams
def test_backward_status_word(i8):
    M, N, K = 300, 520, 1040
    CB, SCB, _ = i8.i8_quantize_rowwise(dev(wl.weight(11, N, K)), 0.0)
    dY = dev(wl.grad_output(12, M, N))
    Wt = i8.i8_dequant_transposed(CB, SCB)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    a = i8.i8_linear8bit_backward_input(dY, Wt, status=status)
    b = i8.i8_linear8bit_backward_input(dY, Wt)
    assert int(host(status)[0]) == 0
    assert torch.equal(a, b)


@pytest.mark.parametrize("M,N,K,n_out", [(512, 1024, 2048, 4), (16, 4096, 8192, 8)])
def test_forwards_on_two_streams(i8, M, N, K, n_out):
    """Two streams of one device run forwards at once (each with its own workspace and
    output); every output equals the same forward run alone."""
    cases = []
    for s in range(2):
        X, _ = wl.activation(wl.BASE_SEED + 500 + s, M, K, n_out, (20.0, 60.0))
        CB, SCB, _ = i8.i8_quantize_rowwise(dev(wl.weight(510 + s, N, K)), 0.0)
        b = dev(wl.bias(520 + s, N))
        ref, _ = i8.i8_linear8bit_forward(dev(X), CB, SCB, b, 6.0)
        cases.append((dev(X), CB, SCB, b, ref.clone()))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [[None] * 10 for _ in range(2)]
    wss = []
    for s in range(2):
        with torch.cuda.stream(streams[s]):
            X, CB, SCB, b, _ = cases[s]
            wss.append(torch.empty((i8.i8_linear8bit_workspace_size(M, N, K, 256),), dtype=torch.uint8, device="cuda"))
    for k in range(10):
        for s in range(2):
            with torch.cuda.stream(streams[s]):
                X, CB, SCB, b, _ = cases[s]
                outs[s][k] = torch.empty((M, N), dtype=torch.float16, device="cuda")
                i8.i8_linear8bit_forward(X, CB, SCB, b, 6.0, out=outs[s][k], workspace=wss[s])
    torch.cuda.synchronize()
    for s in range(2):
        with torch.cuda.stream(streams[s]):
            assert i8.i8_read_status(wss[s]) == (0, n_out)
        for k in range(10):
            assert torch.equal(outs[s][k], cases[s][4]), (s, k)
