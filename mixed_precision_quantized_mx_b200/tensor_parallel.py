"""Output-feature sharding of the layer over ranks (tensor parallelism along N).

The rows of W are independent sub-problems (MixLLM section 3.1.1, Figure 1, and
section 3.3: each output feature needs only its own row, its own quantization and
the activations).  Rank r owns the contiguous rows [start_r, stop_r) of W: it packs
them with the slice of the layer's 8-bit mask, so every row keeps the precision the
global selection gave it, under a permutation local to the rank, and computes
Y[:, start_r:stop_r] with mx_linear on its own GPU.  The only exchange is one
all-gather of Y along N (2 M N bytes in all, against the weights, which never cross
ranks).  The gathered Y is the single-GPU result column for column: each column is
computed from the same row, codes and scales.

One process per GPU, torch.distributed for the plumbing (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(N: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [start, stop) of rank `rank`: contiguous, the first N % world ranks one row more."""
    if world < 1 or not 0 <= rank < world or N < 0:
        raise ValueError(f"N={N} world={world} rank={rank}")
    base, rem = divmod(N, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


def gather_columns(y_local: torch.Tensor, N: int, world: int, group=None) -> torch.Tensor:
    """Y [M, N] from every rank's columns [M, stop_r - start_r] (this rank's is y_local):
    one all-gather of equal-sized blocks (the shards padded to the largest), then the
    columns put back in rank order."""
    if world == 1:
        return y_local
    M = y_local.shape[0]
    width = -(-N // world)
    block = y_local.new_zeros((M, width))
    block[:, :y_local.shape[1]] = y_local
    blocks = [torch.empty_like(block) for _ in range(world)]
    dist.all_gather(blocks, block, group=group)
    cols = []
    for r in range(world):
        a, b = shard_range(N, world, r)
        cols.append(blocks[r][:, :b - a])
    return torch.cat(cols, dim=1)


class ShardedLinear:
    """Y = X W^T with W's output features split over the ranks of a process group.

    W: the layer's full weights [N, K] (host or device; only this rank's rows are
    copied to its GPU) or, with local=True, this rank's rows already sliced.  is8: the
    layer's full 8-bit mask [N] (the result of the global selection).
    """

    def __init__(self, W: torch.Tensor, is8: torch.Tensor, group: int = 128, N: int | None = None,
                 local: bool = False, process_group=None, device=None):
        from .layer import MixedPrecisionLinear
        self.pg = process_group
        distributed = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(process_group) if distributed else 1
        self.rank = dist.get_rank(process_group) if distributed else 0
        self.N = int(N if N is not None else (is8.shape[0] if not local else W.shape[0]))
        self.start, self.stop = shard_range(self.N, self.world, self.rank)
        W_r = W if local else W[self.start:self.stop]
        if W_r.shape[0] != self.stop - self.start:
            raise ValueError(f"rank {self.rank} holds {W_r.shape[0]} rows, its shard has {self.stop - self.start}")
        is8_r = is8[self.start:self.stop] if is8.shape[0] == self.N else is8
        device = device or torch.device("cuda", torch.cuda.current_device())
        self.layer = MixedPrecisionLinear(W_r.to(device), is8_r.to(device, torch.uint8), group)

    def forward(self, X: torch.Tensor) -> torch.Tensor:
        """X [M, K] on this rank's GPU (every rank the same tokens); returns Y [M, N]."""
        return gather_columns(self.layer(X), self.N, self.world, self.pg)

    __call__ = forward
