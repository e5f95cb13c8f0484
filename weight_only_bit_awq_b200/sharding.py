"""Column-parallel (N-sharded) W4A16 linear layer across ranks.

Output channels are independent, so a layer shards over its N output
channels with no exchange in the matmul itself: rank r holds the packed
weights of channels [n0, n1) and computes y[:, n0:n1]. Shard boundaries fall
on whole groups of 128 channels (8 row blocks of the packed layout, which
awq_pack stores one after another), so a rank's packed buffers are exactly
what awq_pack writes for its slice W[n0:n1] of the weight, and its scale and
zero-point columns are the matching column slices. When the caller needs the
full y on every rank, one all-gather of the M x N fp16 output assembles it
(torch.distributed: NCCL on GPUs, gloo on CPUs).

This module is host logic only: the matmul of a shard runs in the library's
CUDA kernels (see ``ShardedLinear``); ``all_gather_columns`` takes any
per-rank slice, so the assembly can be exercised without a GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

SHARD_ALIGN = 128  # output channels per group of 8 row blocks in the packed layout


def shard_range(N: int, world: int, rank: int, align: int = SHARD_ALIGN) -> tuple[int, int]:
    """Output channels [n0, n1) of `rank` out of `world`: contiguous whole
    groups of `align` channels, as equal as possible, lower ranks taking the
    extra groups; the last group may be partial (N % 16 == 0 is required by the
    packed layout, not N % 128). A rank may get an empty range when N has
    fewer groups than there are ranks."""
    if N <= 0 or N % 16 != 0:
        raise ValueError("N must be a positive multiple of 16")
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    groups = (N + align - 1) // align
    base, extra = divmod(groups, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    return min(g0 * align, N), min(g1 * align, N)


def max_shard(N: int, world: int, align: int = SHARD_ALIGN) -> int:
    return max(n1 - n0 for n0, n1 in (shard_range(N, world, r, align) for r in range(world)))


def all_gather_columns(y_local: torch.Tensor, N: int, world: int, rank: int, group=None,
                       align: int = SHARD_ALIGN) -> torch.Tensor:
    """[M, n1 - n0] slice of this rank -> [M, N] on every rank. Slices are
    padded to the largest shard so every rank sends the same number of bytes
    (one all-gather), then placed at their channel offsets."""
    M = y_local.shape[0]
    n0, n1 = shard_range(N, world, rank, align)
    if y_local.shape[1] != n1 - n0:
        raise ValueError(f"rank {rank} slice must have {n1 - n0} columns")
    w = max_shard(N, world, align)
    send = torch.zeros((M, w), dtype=y_local.dtype, device=y_local.device)
    send[:, : n1 - n0] = y_local
    parts = [torch.empty_like(send) for _ in range(world)]
    if world == 1:
        parts[0].copy_(send)
    else:
        dist.all_gather(parts, send.contiguous(), group=group)
    out = torch.empty((M, N), dtype=y_local.dtype, device=y_local.device)
    for r in range(world):
        a, b = shard_range(N, world, r, align)
        out[:, a:b] = parts[r][:, : b - a]
    return out


class ShardedLinear:
    """One rank's shard of a W4A16 layer: packs W[n0:n1] on this GPU with
    awq_pack and runs awq_linear on it; ``forward`` returns the local slice,
    ``forward_full`` the all-gathered [M, N] output."""

    def __init__(self, W: torch.Tensor, world: int, rank: int, group_size: int = 128, pg=None):
        import weight_only_bit_awq_b200 as awq

        self.awq = awq
        self.N, self.K = W.shape
        self.world, self.rank, self.group_size, self.pg = world, rank, group_size, pg
        self.n0, self.n1 = shard_range(self.N, world, rank)
        self.n_local = self.n1 - self.n0
        dev = W.device
        self.ws = awq.new_workspace(awq.GEMV_MAX_M, self.K, max(self.n_local, 16), dev, group_size)
        self.packed = None
        if self.n_local:
            self.packed = awq.awq_pack(W[self.n0:self.n1].contiguous(), self.ws, group_size)
            st = awq.awq_get_status(self.ws)
            if st != awq.AWQ_OK:
                raise RuntimeError(awq.awq_status_string(st))

    def workspace_for(self, M: int) -> torch.Tensor:
        need = self.awq.awq_workspace_bytes(M, self.K, max(self.n_local, 16), self.group_size)
        if self.ws.numel() < need:
            self.ws = self.awq.new_workspace(M, self.K, max(self.n_local, 16), self.ws.device, self.group_size)
        return self.ws

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None) -> torch.Tensor:
        M = x.shape[0]
        if not self.n_local:
            return torch.empty((M, 0), dtype=torch.float16, device=x.device)
        return self.awq.awq_linear(x, *self.packed, self.n_local, self.workspace_for(M), self.group_size, y=y)

    def forward_full(self, x: torch.Tensor) -> torch.Tensor:
        return all_gather_columns(self.forward(x), self.N, self.world, self.rank, self.pg)
