"""Host-side checks of the C ABI: the library builds and loads, exports every
entry point include/i8lt.h declares, and rejects bad arguments before touching
the device (so these run without a GPU)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "i8lt.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"I8_API\s+[\w\s\*]+?\b(i8_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from int8_mixed_precision_vectorwise_b200 import build, _binding
    build.build()
    return _binding.lib()


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for must in ("i8_quantize_rowwise", "i8_linear8bit_forward", "i8_dequant", "i8_int8_linear_matmul",
                 "i8_int8_mm_dequant", "i8_read_status", "i8_dequant_transposed",
                 "i8_linear8bit_backward_input"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    from int8_mixed_precision_vectorwise_b200 import _binding
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    assert sorted(_binding.EXPORTS) == names


def test_status_strings(lib):
    for code, name in [(0, b"I8_OK"), (1, b"I8_ERR_INVALID_ARG"), (6, b"I8_ERR_OUTLIER_OVERFLOW"),
                       (99, b"I8_ERR_UNKNOWN")]:
        assert lib.i8_status_string(code) == name


def test_workspace_size_is_host_only(lib):
    n0 = lib.i8_linear8bit_workspace_size(4096, 4096, 4096, 0)
    n1 = lib.i8_linear8bit_workspace_size(4096, 4096, 4096, 64)
    assert n0 >= 4096 * 4096 + 4096 * 4
    # the gathered outlier operands add (M + N) * 64 fp16
    assert n1 - n0 >= (4096 + 4096) * 64 * 2
    assert lib.i8_linear8bit_workspace_size(0, 4, 16, 0) == 0
    assert lib.i8_linear8bit_workspace_size(4, 4, 16, 100000) == 0


FAKE = ctypes.c_void_p(0x1000)       # never dereferenced: validation fails first
FAKE_MIS = ctypes.c_void_p(0x1008)   # 8-byte aligned only


def test_quantize_rejects(lib):
    f = lib.i8_quantize_rowwise
    assert f(None, 4, 16, 0.0, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 0, 16, 0.0, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 4, 16, -1.0, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 4, 16, float("nan"), FAKE, FAKE, None, None) == 1
    assert f(FAKE, 4, 16, 6.0, FAKE, FAKE, None, None) == 1       # bitmap required
    assert f(FAKE, 4, 24, 0.0, FAKE, FAKE, None, None) == 2       # K % 16
    assert f(FAKE_MIS, 4, 16, 0.0, FAKE, FAKE, None, None) == 2   # alignment


def test_matmul_rejects(lib):
    f = lib.i8_int8_linear_matmul
    assert f(None, FAKE, 4, 4, 16, FAKE, None) == 1
    assert f(FAKE, FAKE, 4, -1, 16, FAKE, None) == 1
    assert f(FAKE, FAKE, 4, 4, 40, FAKE, None) == 2
    assert f(FAKE, FAKE, 4, 4, 16, None, None) == 1
    assert f(FAKE, FAKE, 4, 4, 16, FAKE_MIS, None) == 2


def test_forward_rejects(lib):
    f = lib.i8_linear8bit_forward
    n = lib.i8_linear8bit_workspace_size(4, 4, 16, 8)
    assert f(FAKE, FAKE, FAKE, None, 4, 4, 16, 6.0, FAKE, None, n, 8, None) == 1
    assert f(FAKE, FAKE, None, None, 4, 4, 16, 6.0, FAKE, FAKE, n, 8, None) == 1
    assert f(FAKE, FAKE, FAKE, None, 4, 4, 17, 6.0, FAKE, FAKE, n, 8, None) == 2
    assert f(FAKE, FAKE, FAKE, None, 4, 4, 16, -2.0, FAKE, FAKE, n, 8, None) == 1
    assert f(FAKE, FAKE, FAKE, None, 4, 4, 16, 6.0, FAKE, FAKE, n - 1, 8, None) == 3   # too small
    assert f(FAKE, FAKE, FAKE, None, 4, 4, 16, 6.0, FAKE, ctypes.c_void_p(0x1010), n, 8, None) == 3
    assert f(FAKE, FAKE, FAKE, None, 4, 4, 16, 6.0, FAKE, FAKE, n, 100000, None) == 2


def test_other_rejects(lib):
    assert lib.i8_dequant(None, FAKE, 4, 16, FAKE, None) == 1
    assert lib.i8_dequant(FAKE, FAKE, 4, 20, FAKE, None) == 2
    assert lib.i8_int8_mm_dequant(FAKE, FAKE, FAKE, None, 0, 4, FAKE, None) == 1
    assert lib.i8_int8_mm_dequant(FAKE, FAKE, FAKE, FAKE_MIS, 4, 4, FAKE, None) == 2
    assert lib.i8_outlier_columns(None, 16, FAKE, 4, FAKE, None) == 1
    assert lib.i8_outlier_columns(FAKE, 16, None, 4, FAKE, None) == 1
    assert lib.i8_selftest_bounded_wait(FAKE, 10, None) == 1


def test_backward_rejects(lib):
    f = lib.i8_dequant_transposed
    assert f(None, FAKE, 8, 16, FAKE, None) == 1
    assert f(FAKE, FAKE, 0, 16, FAKE, None) == 1
    assert f(FAKE, FAKE, 8, 24, FAKE, None) == 2      # K % 16
    assert f(FAKE, FAKE, 12, 16, FAKE, None) == 2     # N % 8
    assert f(FAKE, FAKE, 8, 16, FAKE_MIS, None) == 2
    g = lib.i8_linear8bit_backward_input
    assert g(None, FAKE, 4, 8, 16, FAKE, None) == 1
    assert g(FAKE, FAKE, 4, 8, 16, None, None) == 1
    assert g(FAKE, FAKE, 4, 0, 16, FAKE, None) == 1
    assert g(FAKE, FAKE, 4, 12, 16, FAKE, None) == 2  # N % 8
    assert g(FAKE, FAKE_MIS, 4, 8, 16, FAKE, None) == 2
    assert lib.i8_read_status(None, None, None) == 1


def test_multi_workspace_and_rejects(lib):
    Ns = (ctypes.c_int * 3)(520, 264, 1040)
    one = (ctypes.c_int * 1)(520)
    f = lib.i8_linear8bit_multi_workspace_size
    f.restype = ctypes.c_size_t
    lib.i8_linear8bit_workspace_size.restype = ctypes.c_size_t
    for M in (7, 300):   # few-token and prefill layouts
        assert f(M, 1040, 1, one, 256) == lib.i8_linear8bit_workspace_size(M, 520, 1040, 256)
        assert f(M, 1040, 3, Ns, 256) > f(M, 1040, 1, one, 256)
    assert f(300, 1040, 0, Ns, 256) == 0
    assert f(300, 1040, 17, Ns, 256) == 0
    assert f(300, 1040, 3, None, 256) == 0
    assert f(300, 1040, 3, (ctypes.c_int * 3)(520, 0, 8), 256) == 0
    g = lib.i8_linear8bit_forward_multi
    P3 = (ctypes.c_void_p * 3)(0x1000, 0x2000, 0x3000)
    n = f(300, 1040, 3, Ns, 256)
    ok = (FAKE, 300, 1040, 3, P3, P3, None, Ns, P3, ctypes.c_float(6.0), FAKE, ctypes.c_size_t(n), 256, None)

    def call(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return g(*a)
    assert call(a0=None) == 1                        # X
    assert call(a3=0) == 1 and call(a3=17) == 1      # G
    assert call(a4=None) == 1 and call(a7=None) == 1 and call(a8=None) == 1
    assert call(a4=(ctypes.c_void_p * 3)(0x1000, None, 0x3000)) == 1   # a null weight
    assert call(a2=1048) == 2                        # K % 16
    assert call(a8=(ctypes.c_void_p * 3)(0x1000, 0x2008, 0x3000)) == 2  # misaligned output
    assert call(a11=ctypes.c_size_t(n - 1)) == 3     # workspace too small
    assert call(a9=ctypes.c_float(-1.0)) == 1



def test_binding_shape_and_device_checks():
    """The binding's buffer checks (shapes, devices, workspace reuse), exercised on CPU tensors:
    the same helpers guard every entry point before a pointer reaches the library."""
    import torch
    from int8_mixed_precision_vectorwise_b200 import _binding as b
    t = torch.zeros((3, 4), dtype=torch.float16)
    b._check_shape(t, (3, 4), "t")
    with pytest.raises(ValueError, match="shape"):
        b._check_shape(t, (4, 3), "t")
    with pytest.raises(ValueError, match="shape"):
        b._check_shape(torch.zeros(12), (3, 4), "t")
    b._check_device(t, torch.device("cpu"), "t")
    with pytest.raises(ValueError, match="must be on"):
        b._check_device(t, torch.device("cuda", 0), "t")
    with pytest.raises(ValueError, match="CUDA"):
        b._arg(t, torch.float16, "t", (3, 4), torch.device("cpu"))       # inputs must live on the GPU
    with pytest.raises(TypeError, match="float16"):
        b._arg(t.float(), torch.float16, "t", (3, 4), torch.device("cpu"))


def test_matmul_ws_size_and_rejects(lib):
    lib.i8_int8_linear_matmul_workspace_size.restype = ctypes.c_size_t
    sz = lib.i8_int8_linear_matmul_workspace_size
    assert sz(17, 4096, 4096) == 0                       # many rows: the tensor-core GEMM needs none
    assert sz(0, 4096, 4096) == 0 and sz(4, -1, 16) == 0
    n16 = sz(16, 28672, 8192)
    # split-K counters (4 per 128-row tile) and the int32 + fp32 partial sums of every slot
    assert n16 >= (28672 // 128) * 4 * 4 + 16 * 28672 * 8
    assert sz(1, 28672, 8192) == n16                      # sized for 16 token columns whatever M is
    f = lib.i8_int8_linear_matmul_ws
    S = ctypes.c_size_t
    assert f(None, FAKE, 4, 4, 16, FAKE, FAKE, S(n16), None, None) == 1
    assert f(FAKE, FAKE, 4, 4, 40, FAKE, FAKE, S(n16), None, None) == 2    # K % 16
    assert f(FAKE, FAKE, 4, 4, 16, None, FAKE, S(n16), None, None) == 1    # C
    need = sz(4, 4, 16)
    assert need > 0
    assert f(FAKE, FAKE, 4, 4, 16, FAKE, None, S(need), None, None) == 3   # few rows need a workspace
    assert f(FAKE, FAKE, 4, 4, 16, FAKE, FAKE, S(need - 1), None, None) == 3
    assert f(FAKE, FAKE, 4, 4, 16, FAKE, ctypes.c_void_p(0x1010), S(need), None, None) == 3
    assert f(FAKE, FAKE, 4, 4, 16, FAKE, FAKE, S(need), ctypes.c_void_p(0x1002), None) == 2  # status alignment


def test_backward_status_rejects(lib):
    g = lib.i8_linear8bit_backward_input_status
    assert g(None, FAKE, 4, 8, 16, FAKE, FAKE, None) == 1
    assert g(FAKE, FAKE, 4, 12, 16, FAKE, FAKE, None) == 2
    assert g(FAKE, FAKE, 4, 8, 16, FAKE, ctypes.c_void_p(0x1001), None) == 2


def test_workspace_layout_matches_size():
    from int8_mixed_precision_vectorwise_b200 import _binding as b
    lib = b.lib()
    lib.i8_linear8bit_workspace_size.restype = ctypes.c_size_t
    for M, N, K, cap in [(1, 28672, 8192, 256), (16, 1024, 1024, 8), (17, 4096, 4096, 256), (300, 520, 1040, 64),
                         (4096, 11008, 4096, 0)]:
        L = b.i8_linear8bit_workspace_layout(M, N, K, cap)
        assert L["total"] == lib.i8_linear8bit_workspace_size(M, N, K, cap)
        assert L["few_tokens"] == int(M <= 16)
        assert L["ld_o"] == (0 if cap == 0 else -(-cap // 64) * 64)
        # regions in order, 256-byte aligned, large enough for what they hold
        order = ["header", "bitmap", "idx", "sca", "ca", "x_o", "w_o"]
        offs = [L[k] for k in order]
        assert all(o % 256 == 0 for o in offs)
        assert offs == sorted(offs)
        assert L["bitmap"] - L["header"] >= 12
        assert L["sca"] - L["idx"] >= 4 * max(cap, 1)
        assert L["ca"] - L["sca"] >= 4 * M
        assert L["x_o"] - L["ca"] >= M * K
        assert L["w_o"] - L["x_o"] >= 2 * M * L["ld_o"]
        if M > 16:
            assert L["total"] - L["w_o"] >= 2 * N * L["ld_o"]
    with pytest.raises(b.I8Error):
        b.i8_linear8bit_workspace_layout(0, 4, 16, 8)
    with pytest.raises(b.I8Error):
        b.i8_linear8bit_workspace_layout(4, 4, 16, 100000)


def test_int8_rounding_by_added_constant_is_round_half_even():
    """The quantiser rounds t = fl32(x * r) by adding 1.5 * 2^23 in fp32 and keeping the low
    byte of the sum's bits.  That byte must be rne(t) (two's complement) for every |t| <= 128:
    ties on a 2^-12 grid, their fp32 neighbours, and random values."""
    import numpy as np
    grid = (np.arange(-128 * 4096, 128 * 4096 + 1, dtype=np.float64) / 4096).astype(np.float32)
    ties = (np.arange(-128, 128, dtype=np.float32) + np.float32(0.5))
    near = np.concatenate([np.nextafter(ties, np.float32(-np.inf)), np.nextafter(ties, np.float32(np.inf))])
    rnd = np.random.default_rng(0).uniform(-128, 128, 1_000_000).astype(np.float32)
    t = np.concatenate([grid, ties, near, rnd, np.float32([0.0, -0.0])])
    s = (t + np.float32(12582912.0)).astype(np.float32)     # one fp32 addition, round to nearest even
    low = (s.view(np.uint32) & np.uint32(0xFF)).astype(np.uint8).view(np.int8)
    want = np.rint(t.astype(np.float64))                     # numpy rint: half to even
    assert np.array_equal(low.astype(np.int64), ((want.astype(np.int64) + 128) % 256) - 128)


def test_nf4_levels_match_oracle_bit_for_bit():
    """The library computes the NF4 levels on the host with its own inverse normal CDF;
    they must equal the oracle's (scipy) values as fp32 bit patterns."""
    import numpy as np
    from int8_mixed_precision_vectorwise_b200 import _binding as b
    from oracle import nf4
    got = np.array(b.i8_nf4_levels(), np.float32)
    assert np.array_equal(got.view(np.uint32), nf4.nf4_levels().view(np.uint32))


def test_nf4_rejects(lib):
    assert lib.i8_nf4_levels(None) == 1
    assert lib.i8_nf4_quantize(None, 4, 64, FAKE, FAKE, None) == 1
    assert lib.i8_nf4_quantize(FAKE, 4, 96, FAKE, FAKE, None) == 2          # K % 64
    assert lib.i8_nf4_gemv(FAKE, 0, FAKE, FAKE, 4, 64, FAKE, None) == 1
    assert lib.i8_nf4_gemv(FAKE, 9, FAKE, FAKE, 4, 64, FAKE, None) == 2      # at most 8 tokens
    assert lib.i8_nf4_gemv(FAKE_MIS, 1, FAKE, FAKE, 4, 64, FAKE, None) == 2
    assert lib.i8_nf4_dequant(FAKE, FAKE, 4, 100, FAKE, None) == 2
