"""Column-parallel LLM.int8() linear over the ranks of a process group (one GPU each).

The layer's output columns are split between ranks (the tensor-parallel split of
a linear layer discussed in exllama issue #95, and the multi-GPU placement of
int8 weights on the `Linear8bitLt` integration page): rank p keeps rows
[p*N/P, (p+1)*N/P) of the int8 weight CB, of its scales SCB and of the bias,
and runs the forward on the whole input X, which every rank holds.

Nothing else has to cross between ranks.  Row-wise weight quantisation acts on
each weight row alone, so a shard of CB is exactly the quantisation of the same
rows of W.  The activation's row scales and outlier columns depend only on X,
which every rank holds, so every rank finds the same ones.  The only exchange
is an all-gather of the output blocks (NCCL over NVLink): it leaves the P
blocks [M, N/P] one after another, and ``i8_gather_column_blocks`` puts them in
place as out [M, N].

The local forward and the reordering run in the library's CUDA kernels; this
module holds the partitioning and the collective call.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding as b


def shard_range(N: int, world: int, rank: int):
    """Output rows [n0, n1) of the weight kept by `rank` (equal contiguous blocks)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a group of {world}")
    if N % world != 0:
        raise ValueError(f"N = {N} does not split into {world} equal column blocks")
    n = N // world
    return rank * n, (rank + 1) * n


def gather_column_blocks(local: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather of every rank's [M, Np] block; returns G [world, M, Np], rank-major."""
    if world == 1:
        return local.unsqueeze(0)
    M, Np = local.shape
    g = torch.empty((world * M, Np), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(g, local.contiguous(), group=group)
    return g.view(world, M, Np)


class ColumnParallelLinear8bit:
    """One Linear8bitLt split by output columns over a process group.

    CB [N, K] int8 and SCB [N] fp32 are the whole quantised weight (from
    ``i8_quantize_rowwise(W, 0)``); each rank keeps its own rows (copied to its
    current device).  ``forward(X)`` takes the replicated X [M, K] and returns the
    whole out [M, N] on every rank.
    """

    def __init__(self, CB, SCB, bias=None, threshold: float = 6.0, max_outlier_cols: int = 256, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.N, self.K = CB.shape
        n0, n1 = shard_range(self.N, self.world, self.rank)
        dev = torch.device("cuda", torch.cuda.current_device())
        self.CB = CB[n0:n1].to(dev).contiguous()
        self.SCB = SCB[n0:n1].to(dev).contiguous()
        self.bias = None if bias is None else bias[n0:n1].to(dev).contiguous()
        self.threshold = float(threshold)
        self.cap = int(max_outlier_cols)
        self._ws = None

    def forward(self, X, out=None):
        M, K = X.shape
        if K != self.K:
            raise ValueError(f"X has {K} features, the weight {self.K}")
        need = b.i8_linear8bit_workspace_size(M, self.CB.shape[0], K, self.cap)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty((need,), dtype=torch.uint8, device=X.device)
        local, _ = b.i8_linear8bit_forward(X, self.CB, self.SCB, self.bias, self.threshold, workspace=self._ws,
                                           max_outlier_cols=self.cap)
        G = gather_column_blocks(local, self.world, self.group)
        return b.i8_gather_column_blocks(G, out)

    __call__ = forward

    def status(self):
        """(status code, outlier columns found) of the last local forward (synchronises)."""
        return b.i8_read_status(self._ws)
