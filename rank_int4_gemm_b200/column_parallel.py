"""Column-parallel (output-channel) split of the layer across ranks.

Y = XW is separable by output column: channel n of Y needs only row n of the
packed weights (Wq, s_w), row n of L2^T, and the whole of X.  So each rank
holds a contiguous slice of the output channels and computes its columns
of Y from the full, replicated X.  Its own activation stage (rotation, the
per-token absmax over the full K, codes, X L1) is the same computation on
every rank, so no collective is needed inside the layer.  The only exchange
is an all-gather of the column slices when the consumer wants the whole Y.

The per-token scales and codes depend only on X, so the gathered Y equals
the one-rank Y exactly (same codes, same integer sums per channel, same
epilogue).  A split along K instead would need the absmax over all of K
before any code exists (a max all-reduce) and a sum all-reduce of partial
outputs afterwards; a split along M is plain data parallelism.
"""
from __future__ import annotations

import torch


def channel_range(N: int, rank: int, world: int) -> tuple[int, int]:
    """[n0, n1) of the output channels owned by `rank`: contiguous, equal
    slices of whole 8-channel groups (the layer's N granularity)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if N % (8 * world) != 0:
        raise ValueError(f"N = {N} does not split into {world} slices of a multiple of 8 channels")
    per = N // world
    return rank * per, (rank + 1) * per


def shard_layer(Wq: torch.Tensor, s_w: torch.Tensor, L2t: torch.Tensor | None, rank: int,
                world: int):
    """This rank's slice of the packed layer: rows [n0, n1) of Wq [N][K/2],
    s_w [N] and L2^T [N][r] (contiguous copies).  L1^T is not split: every
    rank needs X L1 for all of its channels."""
    n0, n1 = channel_range(Wq.shape[0], rank, world)
    sl = slice(n0, n1)
    return (Wq[sl].contiguous(), s_w[sl].contiguous(),
            None if L2t is None else L2t[sl].contiguous())


def gather_columns(Y_local: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather of the ranks' column slices Y_local [M][N/world] into Y
    [M][N] (rank i's slice at columns [i N/world, (i+1) N/world))."""
    import torch.distributed as dist
    if world == 1:
        return Y_local
    Y_local = Y_local.contiguous()
    M, n_loc = Y_local.shape
    parts = torch.empty(world, M, n_loc, dtype=Y_local.dtype, device=Y_local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(parts, Y_local, group=group)
    else:
        dist.all_gather(list(parts.unbind(0)), Y_local, group=group)
    return parts.permute(1, 0, 2).reshape(M, world * n_loc)


def column_parallel_layer(X, L1t, Wq_local, s_w_local, L2t_local, had_block, world, group=None,
                          local_layer=None):
    """One layer split by output columns: this rank's columns from the full
    X (tq_w4a4_lr_layer, or `local_layer` with the same signature), then the
    all-gather.  Every rank returns the whole Y [M][N]."""
    if local_layer is None:
        from .tq import tq_w4a4_lr_layer as local_layer
    Y_local = local_layer(X, L1t, Wq_local, s_w_local, L2t_local, had_block)
    return gather_columns(Y_local, world, group)
