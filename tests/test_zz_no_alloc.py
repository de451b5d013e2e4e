"""The allocation-free forward (built-in scratch) against the workspace forward.

i8_linear8bit_forward_static serves callers that cannot allocate device
memory at the call site (plugin / server hooks handed only a stream, code
under another allocator, loops that must not call cudaMalloc).  It must give
the same outputs as i8_linear8bit_forward, call after call, although every
call reuses the same built-in scratch array.  This file is collected last so
that a stop-at-first-failure run has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 1e-3


@pytest.fixture(scope="module")
def i8():
    from int8_mixed_precision_vectorwise_b200 import build
    build.build()
    import int8_mixed_precision_vectorwise_b200 as m
    m.lib()
    return m


def _host_case(M, N, K, n_out, seed):
    from int8_mixed_precision_vectorwise_b200 import workloads as wl
    X, _ = wl.activation(4321 + seed, M, K, n_out, (20.0, 60.0))
    W = wl.weight(4322 + seed, N, K)
    b = wl.bias(4323 + seed, N)
    return X, W, b


def _case(i8, M, N, K, n_out, seed):
    X, W, b = _host_case(M, N, K, n_out, seed)
    dX, db = torch.from_numpy(X).cuda(), torch.from_numpy(b).cuda()
    CB, SCB, _ = i8.i8_quantize_rowwise(torch.from_numpy(W).cuda(), 0.0)
    return dX, CB, SCB, db


def _static_call(i8, dX, CB, SCB, db, tau, cap, out, status):
    """Call the entry point through the C ABI directly (ctypes on libi8lt.so)."""
    M, K = dX.shape
    N = CB.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return i8.lib().i8_linear8bit_forward_static(P(dX), P(CB), P(SCB), P(db), M, N, K, ctypes.c_float(tau),
                                                 P(out), cap, P(status), stream)


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return bool(np.all(np.abs(a - b) <= ATOL + RTOL * np.abs(b)))


@pytest.mark.parametrize("M,N,K,n_out", [(16, 1024, 1024, 2), (300, 520, 1040, 5), (4, 4096, 8192, 8)])
def test_static_scratch_forward_matches_workspace_forward(i8, M, N, K, n_out):
    import oracle
    X, W, b = _host_case(M, N, K, n_out, seed=M + N)
    dX, db = torch.from_numpy(X).cuda(), torch.from_numpy(b).cuda()
    CB, SCB, _ = i8.i8_quantize_rowwise(torch.from_numpy(W).cuda(), 0.0)
    ref, ws = i8.i8_linear8bit_forward(dX, CB, SCB, db, 6.0, max_outlier_cols=64)
    assert i8.i8_read_status(ws) == (0, n_out)
    rCB, rSCB = oracle.quantize_weight_rowwise(W)
    want = torch.from_numpy(oracle.linear8bit_forward(X, rCB, rSCB, b, 6.0))
    for call in range(2):   # two calls in a row share (and reuse) the built-in scratch
        out = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        status = torch.full((3,), -1, dtype=torch.int32, device="cuda")
        assert _static_call(i8, dX, CB, SCB, db, 6.0, 64, out, status) == 0
        torch.cuda.synchronize()
        assert status.tolist() == [0, n_out, n_out], (call, status.tolist())
        # the same kernels on the same inputs: identical bits to the workspace forward
        assert torch.equal(out, ref), f"call {call} differs from the workspace forward"
        assert _close(out, want), f"call {call} out of tolerance against the oracle"


def test_static_scratch_sequence_leaves_nothing_behind(i8):
    """Calls that leave different contents in the shared scratch, one after another:
    many tokens, few tokens, threshold 0 after threshold 6, an outlier overflow, then a
    normal call.  Each output and status word equals the workspace forward's."""
    seq = [  # M, N, K, planted columns, threshold, capacity
        (300, 520, 1040, 5, 6.0, 64),
        (4, 4096, 8192, 8, 6.0, 64),
        (300, 520, 1040, 5, 0.0, 64),
        (300, 520, 1040, 20, 6.0, 8),     # 20 columns, room for 8: status 6
        (300, 520, 1040, 5, 6.0, 64),
        (16, 1024, 1024, 2, 6.0, 64),
    ]
    for step, (M, N, K, n_out, tau, cap) in enumerate(seq):
        dX, CB, SCB, db = _case(i8, M, N, K, n_out, seed=step)
        ref, ws = i8.i8_linear8bit_forward(dX, CB, SCB, db, tau, max_outlier_cols=cap)
        code, count = i8.i8_read_status(ws)
        out = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        status = torch.full((3,), -1, dtype=torch.int32, device="cuda")
        assert _static_call(i8, dX, CB, SCB, db, tau, cap, out, status) == 0
        torch.cuda.synchronize()
        used = min(count, cap) if tau > 0 else 0
        assert status.tolist() == [code, used, count if tau > 0 else 0], (step, status.tolist())
        if code == 0:
            assert torch.equal(out, ref), f"step {step} differs from the workspace forward"
        else:
            assert code == 6 and count == n_out, (step, code, count)


def test_static_scratch_rejects_oversize(i8):
    dX, CB, SCB, db = _case(i8, 4096, 1024, 16384, 0, seed=7)   # CA alone is 64 MiB > 32 MiB
    out = torch.empty((4096, 1024), dtype=torch.float16, device="cuda")
    status = torch.zeros(3, dtype=torch.int32, device="cuda")
    assert _static_call(i8, dX, CB, SCB, db, 6.0, 64, out, status) == 3   # I8_ERR_WORKSPACE
