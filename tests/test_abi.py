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
