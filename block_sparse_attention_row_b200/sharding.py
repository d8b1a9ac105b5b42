"""Per-head sharding of one layer across ranks (host-side argument logic).

Every (batch, head) of the path is independent in the mask and in the
attention (SpargeAttention2 §2A selects per row; §2C attends per query block
over that row's kept blocks), so a layer splits across GPUs by heads with no
data exchange: rank r of W takes a contiguous range of the flattened B*H
heads and runs the whole path on it. Ranges differ in size by at most one
head. A [B, H, ...] tensor's heads are contiguous in memory, so a rank's
share is a view, and its outputs are the same views of the whole layer's.
"""
from __future__ import annotations

from typing import Tuple

import torch


def head_range(num_heads: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) of the flattened heads that `rank` of `world` takes."""
    if world < 1 or not 0 <= rank < world or num_heads < 0:
        raise ValueError(f"rank {rank} of world {world} over {num_heads} heads")
    base, extra = divmod(num_heads, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def head_shard(X: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """The rank's heads of a contiguous [B, H, ...] tensor, as a [1, hi - lo, ...] view."""
    if not X.is_contiguous() or X.dim() < 2:
        raise ValueError("head_shard needs a contiguous [B, H, ...] tensor")
    B, H = X.shape[:2]
    lo, hi = head_range(B * H, world, rank)
    return X.reshape((1, B * H) + tuple(X.shape[2:]))[:, lo:hi]
