"""A frozen int8 linear layer for repeated forwards: the Linear8bitLt module of
"`bitsandbytes` - `Linear8bitLt` integration into `transformers` models" (the
nn.Linear replacement that keeps int8 weights and runs the mixed int8 / fp16
forward), as a thin holder around ``i8_linear8bit_forward``.

The weight, its row scales and the bias are checked once, when the layer is
built; a call checks only X and the output buffer and reuses one workspace per
token count, so the host cost of a forward is the C entry point and the launch.
Every step of the forward runs in the CUDA library.
"""

from __future__ import annotations

import torch

from . import _binding as _b


class Linear8bitLt:
    """out = X . dequant(CB, SCB)^T + bias with the LLM.int8() mixed decomposition.

    CB [N, K] int8, SCB [N] fp32 and bias [N] fp16 (or None) live on one CUDA device and
    must not be resized or moved while the layer is in use (their storage is read at
    every call; values may change in place)."""

    def __init__(self, CB, SCB, bias=None, threshold: float = 6.0, max_outlier_cols: int = 256):
        _b._need(CB, torch.int8, "CB", 2)
        self.N, self.K = (int(d) for d in CB.shape)
        dev = CB.device
        _b._arg(SCB, torch.float32, "SCB", (self.N,), dev)
        if bias is not None:
            _b._arg(bias, torch.float16, "bias", (self.N,), dev)
        self.CB, self.SCB, self.bias = CB, SCB, bias
        self.device = dev
        self.index = CB.get_device()
        self.threshold = float(threshold)
        self.max_outlier_cols = int(max_outlier_cols)
        self._ptrs = (CB.data_ptr(), SCB.data_ptr(), None if bias is None else bias.data_ptr())
        self._ws = {}
        self.last_workspace = None   # the workspace of the latest call (status word: i8_read_status)

    @classmethod
    def from_weight(cls, W, bias=None, threshold: float = 6.0, max_outlier_cols: int = 256):
        """Quantise an fp16 weight [N, K] row-wise (SCB = rowmax |W|, CB = round(127 W / SCB))."""
        CB, SCB, _ = _b.i8_quantize_rowwise(W, 0.0)
        return cls(CB, SCB, bias, threshold, max_outlier_cols)

    def workspace(self, M: int):
        ws = self._ws.get(M)
        if ws is None:
            need = _b.i8_linear8bit_workspace_size(M, self.N, self.K, self.max_outlier_cols)
            ws = torch.empty((need,), dtype=torch.uint8, device=self.device)
            self._ws[M] = ws
        return ws

    def __call__(self, X, out=None):
        M = X.shape[0] if isinstance(X, torch.Tensor) and X.dim() == 2 else -1
        if not _b._fits(X, torch.float16, (M, self.K), self.index):
            _b._arg(X, torch.float16, "X", (max(M, 0), self.K), self.device)
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.float16, device=self.device)
        elif not _b._fits(out, torch.float16, (M, self.N), self.index):
            _b._arg(out, torch.float16, "out", (M, self.N), self.device)
        ws = self._ws.get(M)
        if ws is None:
            ws = self.workspace(M)
        self.last_workspace = ws
        cb, scb, bias = self._ptrs
        rc = _b.lib().i8_linear8bit_forward(
            X.data_ptr(), cb, scb, bias, M, self.N, self.K, self.threshold, out.data_ptr(),
            ws.data_ptr(), ws.numel(), self.max_outlier_cols, _b._stream_handle(self.index))
        if rc:
            raise _b.I8Error("i8_linear8bit_forward", rc)
        return out
