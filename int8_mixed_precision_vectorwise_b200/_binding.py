"""ctypes binding of ``libi8lt.so`` (the C ABI in ``include/i8lt.h``).

Argument marshalling only: every function checks dtypes / devices / shapes of
torch tensors, allocates missing outputs with torch, and forwards raw device
pointers plus the current CUDA stream to the library.  All arithmetic runs in
the library's CUDA kernels; there is no fallback.  If the library is missing
or cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libi8lt.so")

STATUS = {
    0: "I8_OK",
    1: "I8_ERR_INVALID_ARG",
    2: "I8_ERR_UNSUPPORTED_SHAPE",
    3: "I8_ERR_WORKSPACE",
    4: "I8_ERR_CUDA",
    5: "I8_ERR_TIMEOUT",
    6: "I8_ERR_OUTLIER_OVERFLOW",
}
I8_OK = 0

EXPORTS = (
    "i8_status_string", "i8_quantize_rowwise", "i8_outlier_columns", "i8_int8_linear_matmul",
    "i8_int8_mm_dequant", "i8_dequant", "i8_linear8bit_workspace_size", "i8_linear8bit_forward",
    "i8_read_status", "i8_selftest_bounded_wait", "i8_linear8bit_prepare", "i8_linear8bit_matmul_dequant",
    "i8_linear8bit_forward_static", "i8_dequant_transposed", "i8_linear8bit_backward_input",
    "i8_linear8bit_multi_workspace_size", "i8_linear8bit_forward_multi",
    "i8_int8_linear_matmul_workspace_size", "i8_int8_linear_matmul_ws", "i8_linear8bit_workspace_layout",
    "i8_linear8bit_backward_input_status", "i8_gather_column_blocks",
    "i8_nf4_levels", "i8_nf4_quantize", "i8_nf4_dequant", "i8_nf4_gemv",
)


class WorkspaceLayout(ctypes.Structure):
    """Mirror of ``i8_workspace_layout`` (byte offsets into a forward workspace)."""
    _fields_ = [("header", ctypes.c_size_t), ("bitmap", ctypes.c_size_t), ("idx", ctypes.c_size_t),
                ("sca", ctypes.c_size_t), ("ca", ctypes.c_size_t), ("x_o", ctypes.c_size_t),
                ("w_o", ctypes.c_size_t), ("total", ctypes.c_size_t), ("ld_o", ctypes.c_int),
                ("few_tokens", ctypes.c_int)]


class I8Error(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t


def _declare(lib):
    sig = {
        "i8_status_string": (ctypes.c_char_p, [_I]),
        "i8_quantize_rowwise": (_I, [_P, _I, _I, _F, _P, _P, _P, _P]),
        "i8_outlier_columns": (_I, [_P, _I, _P, _I, _P, _P]),
        "i8_int8_linear_matmul": (_I, [_P, _P, _I, _I, _I, _P, _P]),
        "i8_int8_mm_dequant": (_I, [_P, _P, _P, _P, _I, _I, _P, _P]),
        "i8_dequant": (_I, [_P, _P, _I, _I, _P, _P]),
        "i8_dequant_transposed": (_I, [_P, _P, _I, _I, _P, _P]),
        "i8_gather_column_blocks": (_I, [_P, _I, _I, _I, _P, _P]),
        "i8_nf4_levels": (_I, [_P]),
        "i8_nf4_quantize": (_I, [_P, _I, _I, _P, _P, _P]),
        "i8_nf4_dequant": (_I, [_P, _P, _I, _I, _P, _P]),
        "i8_nf4_gemv": (_I, [_P, _I, _P, _P, _I, _I, _P, _P]),
        "i8_linear8bit_backward_input": (_I, [_P, _P, _I, _I, _I, _P, _P]),
        "i8_linear8bit_multi_workspace_size": (_S, [_I, _I, _I, _P, _I]),
        "i8_linear8bit_forward_multi": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _F, _P, _S, _I, _P]),
        "i8_linear8bit_workspace_size": (_S, [_I, _I, _I, _I]),
        "i8_linear8bit_forward": (_I, [_P, _P, _P, _P, _I, _I, _I, _F, _P, _P, _S, _I, _P]),
        "i8_linear8bit_prepare": (_I, [_P, _P, _I, _I, _I, _F, _P, _S, _I, _P]),
        "i8_linear8bit_matmul_dequant": (_I, [_P, _P, _P, _I, _I, _I, _F, _P, _P, _S, _I, _P]),
        "i8_linear8bit_forward_static": (_I, [_P, _P, _P, _P, _I, _I, _I, _F, _P, _I, _P, _P]),
        "i8_read_status": (_I, [_P, _P, _P]),
        "i8_int8_linear_matmul_workspace_size": (_S, [_I, _I, _I]),
        "i8_int8_linear_matmul_ws": (_I, [_P, _P, _I, _I, _I, _P, _P, _S, _P, _P]),
        "i8_linear8bit_workspace_layout": (_I, [_I, _I, _I, _I, ctypes.POINTER(WorkspaceLayout)]),
        "i8_linear8bit_backward_input_status": (_I, [_P, _P, _I, _I, _I, _P, _P, _P]),
        "i8_selftest_bounded_wait": (_I, [_P, ctypes.c_uint64, _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


def lib():
    """The loaded library (raises if it is not built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m int8_mixed_precision_vectorwise_b200.build`")
                _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def _check(fn: str, code: int):
    if code != I8_OK:
        raise I8Error(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


try:  # the current stream's handle without building a Stream object (a per-call cost)
    _raw_stream = torch._C._cuda_getCurrentRawStream
except AttributeError:  # pragma: no cover - older torch
    def _raw_stream(index):
        return torch.cuda.current_stream(index).cuda_stream


def _stream_handle(index):
    """The current stream of CUDA device `index`, as the integer handle the C ABI takes."""
    return _raw_stream(index)


def _fits(t, dtype, shape, index):
    """True when t is a contiguous CUDA tensor of `dtype` and `shape` on device `index`
    (the cheap test of the per-call path; on False the detailed checks name the problem)."""
    # (get_device() is -1 for a CPU tensor, never a CUDA index)
    return (isinstance(t, torch.Tensor) and t.dtype is dtype and t.get_device() == index
            and t.shape == shape and t.is_contiguous())


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D")


def _check_shape(t, shape, name):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_device(t, dev, name):
    if t.device != dev:
        raise ValueError(f"{name} must be on {dev}, got {t.device}")


def _arg(t, dtype, name, shape, dev):
    """An input the kernels read: dtype, CUDA, contiguous, on `dev`, exactly `shape`."""
    _need(t, dtype, name, len(shape))
    _check_device(t, dev, name)
    _check_shape(t, shape, name)
    return t


def _out(t, dtype, name, shape, dev):
    """A caller-provided buffer the kernels write (checked like an input), or a new one."""
    if t is None:
        return torch.empty(tuple(shape), dtype=dtype, device=dev)
    return _arg(t, dtype, name, shape, dev)


def _workspace(t, dev, need):
    """A caller workspace (uint8, on `dev`) large enough, else a new one."""
    if t is not None:
        _need(t, torch.uint8, "workspace", 1)
        _check_device(t, dev, "workspace")
        if t.numel() >= need:
            return t
    return torch.empty((need,), dtype=torch.uint8, device=dev)


# ----------------------------------------------------------------- entry points
def i8_quantize_rowwise(X, threshold: float = 0.0, CA=None, SCA=None, bitmap=None):
    """Fused row absmax + int8 quantisation + outlier bitmap.  Returns (CA, SCA, bitmap)."""
    _need(X, torch.float16, "X", 2)
    M, K = X.shape
    dev = X.device
    CA = _out(CA, torch.int8, "CA", (M, K), dev)
    SCA = _out(SCA, torch.float32, "SCA", (M,), dev)
    if threshold > 0 or bitmap is not None:
        bitmap = _out(bitmap, torch.int32, "bitmap", ((K + 31) // 32,), dev)
    _check("i8_quantize_rowwise", lib().i8_quantize_rowwise(
        _ptr(X), M, K, float(threshold), _ptr(CA), _ptr(SCA), _ptr(bitmap), _stream(dev)))
    return CA, SCA, bitmap


def i8_outlier_columns(bitmap, K: int, max_cols: int, idx=None, count=None):
    """Sorted outlier column list from a bitmap.  Returns (idx[max_cols], count[1]) on device."""
    _need(bitmap, torch.int32, "bitmap", 1)
    dev = bitmap.device
    _check_shape(bitmap, ((K + 31) // 32,), "bitmap")
    if idx is None:
        idx = torch.empty((max(max_cols, 1),), dtype=torch.int32, device=dev)
    else:
        _need(idx, torch.int32, "idx", 1)
        _check_device(idx, dev, "idx")
        if idx.numel() < max_cols:
            raise ValueError(f"idx must hold max_cols = {max_cols} entries")
    count = _out(count, torch.int32, "count", (1,), dev)
    _check("i8_outlier_columns", lib().i8_outlier_columns(
        _ptr(bitmap), K, _ptr(idx), max_cols, _ptr(count), _stream(dev)))
    return idx, count


def i8_int8_linear_matmul(A, B, C=None):
    """C = A . B^T, int8 x int8 -> int32 (exact)."""
    _need(A, torch.int8, "A", 2)
    _need(B, torch.int8, "B", 2)
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("A and B must share K")
    _check_device(B, A.device, "B")
    C = _out(C, torch.int32, "C", (M, N), A.device)
    _check("i8_int8_linear_matmul", lib().i8_int8_linear_matmul(
        _ptr(A), _ptr(B), M, N, K, _ptr(C), _stream(A.device)))
    return C


def i8_int8_linear_matmul_ws(A, B, C=None, workspace=None, status=None):
    """C = A . B^T (int32, exact) by the kernel the forward uses for these sizes: for at
    most 16 rows of A the few-token stream-K kernel, whose split-K partial sums live in
    `workspace` (allocated here when None).  `status` (int32 [1] on the device, optional)
    receives the device status word.  Returns (C, workspace)."""
    _need(A, torch.int8, "A", 2)
    _need(B, torch.int8, "B", 2)
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("A and B must share K")
    dev = A.device
    _check_device(B, dev, "B")
    C = _out(C, torch.int32, "C", (M, N), dev)
    need = int(lib().i8_int8_linear_matmul_workspace_size(M, N, K))
    workspace = _workspace(workspace, dev, max(need, 1))
    if status is not None:
        _arg(status, torch.int32, "status", (1,), dev)
    _check("i8_int8_linear_matmul_ws", lib().i8_int8_linear_matmul_ws(
        _ptr(A), _ptr(B), M, N, K, _ptr(C), _ptr(workspace), workspace.numel(), _ptr(status), _stream(dev)))
    return C, workspace


def i8_linear8bit_workspace_layout(M: int, N: int, K: int, max_outlier_cols: int) -> dict:
    """Byte offsets of the prepared operands inside a forward workspace (see include/i8lt.h)."""
    lay = WorkspaceLayout()
    _check("i8_linear8bit_workspace_layout",
           lib().i8_linear8bit_workspace_layout(M, N, K, max_outlier_cols, ctypes.byref(lay)))
    return {name: int(getattr(lay, name)) for name, _ in WorkspaceLayout._fields_}


def i8_int8_mm_dequant(C, SCA, SCB, bias=None, out=None):
    """out = fp16(C * SCA[i] * SCB[n] / 127^2 + bias[n])."""
    _need(C, torch.int32, "C", 2)
    M, N = C.shape
    dev = C.device
    _arg(SCA, torch.float32, "SCA", (M,), dev)
    _arg(SCB, torch.float32, "SCB", (N,), dev)
    if bias is not None:
        _arg(bias, torch.float16, "bias", (N,), dev)
    out = _out(out, torch.float16, "out", (M, N), dev)
    _check("i8_int8_mm_dequant", lib().i8_int8_mm_dequant(
        _ptr(C), _ptr(SCA), _ptr(SCB), _ptr(bias), M, N, _ptr(out), _stream(C.device)))
    return out


def i8_dequant(CB, SCB, W=None):
    """W = fp16(CB * SCB[n] / 127)."""
    _need(CB, torch.int8, "CB", 2)
    N, K = CB.shape
    _arg(SCB, torch.float32, "SCB", (N,), CB.device)
    W = _out(W, torch.float16, "W", (N, K), CB.device)
    _check("i8_dequant", lib().i8_dequant(_ptr(CB), _ptr(SCB), N, K, _ptr(W), _stream(CB.device)))
    return W


def i8_dequant_transposed(CB, SCB, Wt=None):
    """Wt = W^T with W = fp16(CB * SCB[n] / 127): CB [N, K] -> Wt [K, N]."""
    _need(CB, torch.int8, "CB", 2)
    N, K = CB.shape
    _arg(SCB, torch.float32, "SCB", (N,), CB.device)
    Wt = _out(Wt, torch.float16, "Wt", (K, N), CB.device)
    _check("i8_dequant_transposed", lib().i8_dequant_transposed(
        _ptr(CB), _ptr(SCB), N, K, _ptr(Wt), _stream(CB.device)))
    return Wt


def i8_gather_column_blocks(G, out=None):
    """out [M, P*Np] from rank-major column blocks G [P, M, Np]: out[m, p*Np + j] = G[p, m, j]."""
    _need(G, torch.float16, "G", 3)
    P, M, Np = G.shape
    out = _out(out, torch.float16, "out", (M, P * Np), G.device)
    _check("i8_gather_column_blocks", lib().i8_gather_column_blocks(
        _ptr(G), P, M, Np, _ptr(out), _stream(G.device)))
    return out


def i8_nf4_levels():
    """The 16 NF4 levels (host, fp32 list, ascending)."""
    buf = (ctypes.c_float * 16)()
    _check("i8_nf4_levels", lib().i8_nf4_levels(buf))
    return list(buf)


def i8_nf4_quantize(W, packed=None, absmax=None):
    """Blockwise (64) NF4 quantisation of an fp16 weight [N, K]: returns (packed [N, K/2] uint8,
    absmax [N, K/64] fp32)."""
    _need(W, torch.float16, "W", 2)
    N, K = W.shape
    packed = _out(packed, torch.uint8, "packed", (N, K // 2), W.device)
    absmax = _out(absmax, torch.float32, "absmax", (N, K // 64), W.device)
    _check("i8_nf4_quantize", lib().i8_nf4_quantize(_ptr(W), N, K, _ptr(packed), _ptr(absmax), _stream(W.device)))
    return packed, absmax


def i8_nf4_dequant(packed, absmax, W=None):
    """fp16 [N, K] dequantised NF4 weight."""
    _need(packed, torch.uint8, "packed", 2)
    N, H = packed.shape
    K = 2 * H
    _arg(absmax, torch.float32, "absmax", (N, K // 64), packed.device)
    W = _out(W, torch.float16, "W", (N, K), packed.device)
    _check("i8_nf4_dequant", lib().i8_nf4_dequant(_ptr(packed), _ptr(absmax), N, K, _ptr(W), _stream(packed.device)))
    return W


def i8_nf4_gemv(X, packed, absmax, out=None):
    """out [M, N] = fp16(X [M, K] . NF4 weight^T), 1 <= M <= 8."""
    _need(X, torch.float16, "X", 2)
    M, K = X.shape
    dev = X.device
    _arg(packed, torch.uint8, "packed", (packed.shape[0], K // 2), dev)
    N = packed.shape[0]
    _arg(absmax, torch.float32, "absmax", (N, K // 64), dev)
    out = _out(out, torch.float16, "out", (M, N), dev)
    _check("i8_nf4_gemv", lib().i8_nf4_gemv(_ptr(X), M, _ptr(packed), _ptr(absmax), N, K, _ptr(out), _stream(dev)))
    return out


def i8_linear8bit_backward_input(dY, Wt, dX=None, status=None):
    """dX = fp16(dY . Wt^T): dY [M, N], Wt [K, N] (from i8_dequant_transposed) -> dX [M, K].
    `status` (int32 [1] on the device, optional) receives the device status word."""
    _need(dY, torch.float16, "dY", 2)
    _need(Wt, torch.float16, "Wt", 2)
    M, N = dY.shape
    K = Wt.shape[0]
    if Wt.shape[1] != N:
        raise ValueError("dY and Wt must share N")
    _check_device(Wt, dY.device, "Wt")
    dX = _out(dX, torch.float16, "dX", (M, K), dY.device)
    if status is None:
        _check("i8_linear8bit_backward_input", lib().i8_linear8bit_backward_input(
            _ptr(dY), _ptr(Wt), M, N, K, _ptr(dX), _stream(dY.device)))
    else:
        _arg(status, torch.int32, "status", (1,), dY.device)
        _check("i8_linear8bit_backward_input_status", lib().i8_linear8bit_backward_input_status(
            _ptr(dY), _ptr(Wt), M, N, K, _ptr(dX), _ptr(status), _stream(dY.device)))
    return dX


_ws_sizes: dict = {}


def i8_linear8bit_workspace_size(M: int, N: int, K: int, max_outlier_cols: int) -> int:
    key = (id(lib()), M, N, K, max_outlier_cols)   # remembered per shape (a per-call cost otherwise)
    n = _ws_sizes.get(key)
    if n is None:
        n = int(lib().i8_linear8bit_workspace_size(M, N, K, max_outlier_cols))
        if n == 0:
            raise I8Error("i8_linear8bit_workspace_size", 1)
        if len(_ws_sizes) < 4096:
            _ws_sizes[key] = n
    return n


def i8_linear8bit_forward(X, CB, SCB, bias=None, threshold: float = 6.0, out=None, workspace=None,
                          max_outlier_cols: int = 256):
    """LLM.int8() Linear8bitLt forward.  Returns (out, workspace)."""
    _need(X, torch.float16, "X", 2)
    M, K = X.shape
    dev = X.device
    index = X.get_device()
    N = CB.shape[0] if isinstance(CB, torch.Tensor) and CB.dim() == 2 else -1
    need = i8_linear8bit_workspace_size(M, N, K, max_outlier_cols) if N > 0 else 0
    if not (_fits(CB, torch.int8, (N, K), index) and _fits(SCB, torch.float32, (N,), index)
            and (bias is None or _fits(bias, torch.float16, (N,), index))
            and (out is None or _fits(out, torch.float16, (M, N), index))
            and (workspace is None or (_fits(workspace, torch.uint8, workspace.shape, index)
                                       and workspace.dim() == 1))):
        # the detailed checks raise with a message naming the argument
        _need(CB, torch.int8, "CB", 2)
        _arg(CB, torch.int8, "CB", (N, K), dev)
        _arg(SCB, torch.float32, "SCB", (N,), dev)
        if bias is not None:
            _arg(bias, torch.float16, "bias", (N,), dev)
        if out is not None:
            _out(out, torch.float16, "out", (M, N), dev)
        if workspace is not None:
            _workspace(workspace, dev, need)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
    _check("i8_linear8bit_forward", lib().i8_linear8bit_forward(
        X.data_ptr(), CB.data_ptr(), SCB.data_ptr(), None if bias is None else bias.data_ptr(), M, N, K,
        float(threshold), out.data_ptr(), workspace.data_ptr(), workspace.numel(), max_outlier_cols,
        _stream_handle(index)))
    return out, workspace


def _ptr_array(ts):
    return (ctypes.c_void_p * len(ts))(*[None if t is None else t.data_ptr() for t in ts])


def i8_linear8bit_multi_workspace_size(M: int, K: int, Ns, max_outlier_cols: int) -> int:
    arr = (ctypes.c_int * len(Ns))(*Ns)
    n = lib().i8_linear8bit_multi_workspace_size(M, K, len(Ns), arr, max_outlier_cols)
    if n == 0:
        raise I8Error("i8_linear8bit_multi_workspace_size", 1)
    return int(n)


def i8_linear8bit_forward_multi(X, CBs, SCBs, biases=None, threshold: float = 6.0, outs=None, workspace=None,
                                max_outlier_cols: int = 256):
    """Forward of several weights over the same X (X quantised once).  Returns (outs, workspace)."""
    _need(X, torch.float16, "X", 2)
    G = len(CBs)
    if len(SCBs) != G or (biases is not None and len(biases) != G) or (outs is not None and len(outs) != G):
        raise ValueError("CBs, SCBs, biases and outs must have one entry per weight")
    biases = [None] * G if biases is None else list(biases)
    M, K = X.shape
    dev = X.device
    for g in range(G):
        _need(CBs[g], torch.int8, "CB", 2)
        N = CBs[g].shape[0]
        _arg(CBs[g], torch.int8, "CB", (N, K), dev)
        _arg(SCBs[g], torch.float32, "SCB", (N,), dev)
        if biases[g] is not None:
            _arg(biases[g], torch.float16, "bias", (N,), dev)
    Ns = [int(CB.shape[0]) for CB in CBs]
    workspace = _workspace(workspace, dev, i8_linear8bit_multi_workspace_size(M, K, Ns, max_outlier_cols))
    outs = [_out(None if outs is None else outs[g], torch.float16, "out", (M, Ns[g]), dev) for g in range(G)]
    n_arr = (ctypes.c_int * G)(*Ns)
    _check("i8_linear8bit_forward_multi", lib().i8_linear8bit_forward_multi(
        _ptr(X), M, K, G, _ptr_array(CBs), _ptr_array(SCBs), _ptr_array(biases), n_arr, _ptr_array(outs),
        float(threshold), _ptr(workspace), workspace.numel(), max_outlier_cols, _stream(dev)))
    return outs, workspace


def i8_linear8bit_prepare(X, CB, threshold: float, workspace, max_outlier_cols: int = 256):
    """First half of the forward: quantise X and prepare the outlier operands in `workspace`."""
    _need(X, torch.float16, "X", 2)
    M, K = X.shape
    _need(CB, torch.int8, "CB", 2)
    N = CB.shape[0]
    _arg(CB, torch.int8, "CB", (N, K), X.device)
    _need(workspace, torch.uint8, "workspace", 1)
    _check_device(workspace, X.device, "workspace")
    _check("i8_linear8bit_prepare", lib().i8_linear8bit_prepare(
        _ptr(X), _ptr(CB), M, N, K, float(threshold), _ptr(workspace), workspace.numel(),
        max_outlier_cols, _stream(X.device)))


def i8_linear8bit_matmul_dequant(CB, SCB, bias, M: int, threshold: float, out, workspace,
                                 max_outlier_cols: int = 256):
    """Second half of the forward: the tensor-core GEMM with the fused epilogue."""
    _need(CB, torch.int8, "CB", 2)
    N, K = CB.shape
    dev = CB.device
    _arg(SCB, torch.float32, "SCB", (N,), dev)
    if bias is not None:
        _arg(bias, torch.float16, "bias", (N,), dev)
    _arg(out, torch.float16, "out", (M, N), dev)
    _need(workspace, torch.uint8, "workspace", 1)
    _check_device(workspace, dev, "workspace")
    _check("i8_linear8bit_matmul_dequant", lib().i8_linear8bit_matmul_dequant(
        _ptr(CB), _ptr(SCB), _ptr(bias), M, N, K, float(threshold), _ptr(out), _ptr(workspace),
        workspace.numel(), max_outlier_cols, _stream(CB.device)))
    return out


def i8_linear8bit_forward_static(X, CB, SCB, bias=None, threshold: float = 6.0, out=None,
                                 max_outlier_cols: int = 256, status_out=None):
    """Forward using the library's built-in scratch instead of a workspace (see include/i8lt.h)."""
    _need(X, torch.float16, "X", 2)
    M, K = X.shape
    dev = X.device
    _need(CB, torch.int8, "CB", 2)
    N = CB.shape[0]
    _arg(CB, torch.int8, "CB", (N, K), dev)
    _arg(SCB, torch.float32, "SCB", (N,), dev)
    if bias is not None:
        _arg(bias, torch.float16, "bias", (N,), dev)
    out = _out(out, torch.float16, "out", (M, N), dev)
    if status_out is not None:
        _need(status_out, torch.int32, "status_out", 1)
        _check_device(status_out, dev, "status_out")
        if status_out.numel() < 3:
            raise ValueError("status_out must hold 3 words")
    _check("i8_linear8bit_forward_static", lib().i8_linear8bit_forward_static(
        _ptr(X), _ptr(CB), _ptr(SCB), _ptr(bias), M, N, K, float(threshold), _ptr(out), max_outlier_cols,
        _ptr(status_out), _stream(X.device)))
    return out


def i8_read_status(workspace):
    """Synchronise the current stream; returns (status_code, outlier_count) of the last forward."""
    cnt = ctypes.c_int32(0)
    code = lib().i8_read_status(_ptr(workspace), ctypes.byref(cnt), _stream(workspace.device))
    return int(code), int(cnt.value)


def i8_selftest_bounded_wait(status, limit_ns: int):
    _need(status, torch.int32, "status", 1)
    _check("i8_selftest_bounded_wait", lib().i8_selftest_bounded_wait(
        _ptr(status), int(limit_ns), _stream(status.device)))
    return status
