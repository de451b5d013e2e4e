"""The Python binding's argument marshalling, on CPU.

Every wrapper is called with CPU tensors against a stand-in for the library
that records its arguments and returns I8_OK.  Only the CUDA-residency test and
the stream lookup are relaxed for this; shapes, dtypes, devices, output
allocation, workspace reuse and the integer sizes handed to the C ABI are the
binding's own.
"""
import pytest
import torch

from int8_mixed_precision_vectorwise_b200 import _binding as b


class FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("i8_"):
            raise AttributeError(name)

        def fn(*args):
            self.calls.append((name, args))
            return 4096 if name.endswith("workspace_size") else 0
        return fn


@pytest.fixture()
def fake(monkeypatch):
    lib = FakeLib()
    real_need = b._need

    def need_on_any_device(t, dtype, name, ndim=None):
        if isinstance(t, torch.Tensor) and not t.is_cuda:
            # same checks, CUDA residency aside
            if t.dtype != dtype:
                raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
            if not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous")
            if ndim is not None and t.dim() != ndim:
                raise ValueError(f"{name} must be {ndim}-D")
            return
        real_need(t, dtype, name, ndim)

    monkeypatch.setattr(b, "_need", need_on_any_device)
    monkeypatch.setattr(b, "_stream", lambda dev: None)
    monkeypatch.setattr(b, "_stream_handle", lambda index: None)
    monkeypatch.setattr(b, "lib", lambda: lib)
    return lib


def z(shape, dtype):
    return torch.zeros(shape, dtype=dtype)


def test_forward_shapes_and_sizes(fake):
    M, N, K = 5, 24, 32
    X, CB, SCB, bias = z((M, K), torch.float16), z((N, K), torch.int8), z(N, torch.float32), z(N, torch.float16)
    out, ws = b.i8_linear8bit_forward(X, CB, SCB, bias, 6.0)
    assert out.shape == (M, N) and out.dtype == torch.float16 and ws.numel() == 4096
    name, args = fake.calls[-1]
    assert name == "i8_linear8bit_forward" and args[4:8] == (M, N, K, 6.0)
    out2, ws2 = b.i8_linear8bit_forward(X, CB, SCB, None, 6.0, out=out, workspace=ws)
    assert out2 is out and ws2 is ws                       # caller buffers are used as given
    with pytest.raises(ValueError, match="shape"):
        b.i8_linear8bit_forward(X, CB, z(N + 1, torch.float32), None)
    with pytest.raises(ValueError, match="shape"):
        b.i8_linear8bit_forward(X, CB, SCB, z(N - 1, torch.float16))
    with pytest.raises(ValueError, match="shape"):
        b.i8_linear8bit_forward(X, CB, SCB, None, out=z((M, N + 8), torch.float16))
    with pytest.raises(ValueError, match="shape"):
        b.i8_linear8bit_forward(X, z((N, K + 16), torch.int8), SCB)
    with pytest.raises(TypeError):
        b.i8_linear8bit_forward(X, CB, SCB, None, workspace=z(4096, torch.int32))
    small = z(16, torch.uint8)
    _, ws3 = b.i8_linear8bit_forward(X, CB, SCB, None, workspace=small)
    assert ws3 is not small and ws3.numel() == 4096      # too small: a new one is allocated


def test_split_forward_and_static(fake):
    M, N, K = 3, 16, 48
    X, CB, SCB = z((M, K), torch.float16), z((N, K), torch.int8), z(N, torch.float32)
    ws = z(4096, torch.uint8)
    b.i8_linear8bit_prepare(X, CB, 6.0, ws)
    out = z((M, N), torch.float16)
    assert b.i8_linear8bit_matmul_dequant(CB, SCB, None, M, 6.0, out, ws) is out
    with pytest.raises(ValueError, match="shape"):
        b.i8_linear8bit_matmul_dequant(CB, SCB, None, M + 1, 6.0, out, ws)
    assert b.i8_linear8bit_forward_static(X, CB, SCB).shape == (M, N)
    b.i8_linear8bit_forward_static(X, CB, SCB, status_out=z(3, torch.int32))
    with pytest.raises(ValueError, match="3 words"):
        b.i8_linear8bit_forward_static(X, CB, SCB, status_out=z(2, torch.int32))


def test_multi_forward(fake):
    M, K, Ns = 7, 64, (40, 8, 24)
    X = z((M, K), torch.float16)
    CBs = [z((n, K), torch.int8) for n in Ns]
    SCBs = [z(n, torch.float32) for n in Ns]
    outs, ws = b.i8_linear8bit_forward_multi(X, CBs, SCBs, [z(40, torch.float16), None, None], 6.0)
    assert [tuple(o.shape) for o in outs] == [(M, n) for n in Ns]
    name, args = fake.calls[-1]
    assert name == "i8_linear8bit_forward_multi" and args[1:4] == (M, K, 3)
    assert list(args[7]) == list(Ns)
    given = [z((M, n), torch.float16) for n in Ns]
    outs2, _ = b.i8_linear8bit_forward_multi(X, CBs, SCBs, None, 6.0, outs=given, workspace=ws)
    assert all(a is c for a, c in zip(outs2, given))
    with pytest.raises(ValueError, match="one entry per weight"):
        b.i8_linear8bit_forward_multi(X, CBs, SCBs[:2])
    with pytest.raises(ValueError, match="shape"):
        b.i8_linear8bit_forward_multi(X, CBs, SCBs, None, 6.0, outs=given[:2] + [z((M, 8), torch.float16)])


def test_other_ops(fake):
    M, N, K = 4, 16, 32
    CA, SCA, bm = b.i8_quantize_rowwise(z((M, K), torch.float16), 6.0)
    assert CA.shape == (M, K) and SCA.shape == (M,) and bm.shape == (1,)
    assert b.i8_quantize_rowwise(z((M, K), torch.float16), 0.0)[2] is None
    idx, cnt = b.i8_outlier_columns(bm, K, 8)
    assert idx.shape == (8,) and cnt.shape == (1,)
    with pytest.raises(ValueError, match="shape"):
        b.i8_outlier_columns(z(2, torch.int32), K, 8)
    C = b.i8_int8_linear_matmul(z((M, K), torch.int8), z((N, K), torch.int8))
    assert C.shape == (M, N) and C.dtype == torch.int32
    out = b.i8_int8_mm_dequant(C, z(M, torch.float32), z(N, torch.float32))
    assert out.shape == (M, N)
    with pytest.raises(ValueError, match="shape"):
        b.i8_int8_mm_dequant(C, z(N, torch.float32), z(N, torch.float32))
    CB, SCB = z((N, K), torch.int8), z(N, torch.float32)
    assert b.i8_dequant(CB, SCB).shape == (N, K)
    Wt = b.i8_dequant_transposed(CB, SCB)
    assert Wt.shape == (K, N)
    dX = b.i8_linear8bit_backward_input(z((M, N), torch.float16), Wt)
    assert dX.shape == (M, K)
    with pytest.raises(ValueError, match="shape"):
        b.i8_linear8bit_backward_input(z((M, N), torch.float16), Wt, dX=z((M, K + 1), torch.float16))


def test_layer_checks_weights_once_and_x_per_call(fake):
    from int8_mixed_precision_vectorwise_b200.layer import Linear8bitLt
    N, K = 24, 32
    CB, SCB, bias = z((N, K), torch.int8), z(N, torch.float32), z(N, torch.float16)
    layer = Linear8bitLt(CB, SCB, bias, threshold=6.0)
    out = layer(z((5, K), torch.float16))
    assert out.shape == (5, N) and out.dtype == torch.float16
    name, args = fake.calls[-1]
    assert name == "i8_linear8bit_forward" and args[4:8] == (5, N, K, 6.0)
    assert args[1] == CB.data_ptr() and args[3] == bias.data_ptr()
    ws5 = layer.workspace(5)
    buf = z((3, N), torch.float16)
    assert layer(z((3, K), torch.float16), out=buf) is buf       # a caller buffer is used as given
    layer(z((5, K), torch.float16))
    assert layer.workspace(5) is ws5                             # one workspace per token count
    with pytest.raises(ValueError, match="shape"):
        layer(z((5, K + 16), torch.float16))
    with pytest.raises(TypeError):
        layer(z((5, K), torch.float32))
    with pytest.raises(ValueError, match="shape"):
        layer(z((5, K), torch.float16), out=z((5, N + 8), torch.float16))
    with pytest.raises(ValueError, match="shape"):
        Linear8bitLt(CB, z(N + 1, torch.float32))
