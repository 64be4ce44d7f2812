"""Output-channel (N) sharding of the layer over ranks, one GPU per rank.

Every rank holds the rows [n0, n1) of W (CB, SCB, the optional fp16 weight and
the bias) and the whole of X. The outlier set O depends on X alone, so every
rank derives the same O, the same CA and SCA, and computes its columns of
Y = X W^T + bias exactly as the unsharded layer would: the forward needs no
collective. An all-gather of the shards is only needed when every rank wants
the whole of Y.

Shards are contiguous, a multiple of 32 output channels each (the row block of
the blocked weight layout), the last one possibly shorter or empty.
"""
from __future__ import annotations


def shard_rows(N: int, world: int, rank: int, align: int = 32) -> tuple[int, int]:
    """Rows [n0, n1) of an N-row weight that rank `rank` of `world` holds."""
    if world < 1 or not 0 <= rank < world or N < 0:
        raise ValueError(f"bad shard request N={N} world={world} rank={rank}")
    per = -(-N // world)
    per = -(-per // align) * align
    n0 = min(N, rank * per)
    return n0, min(N, n0 + per)


def shard_width(N: int, world: int, align: int = 32) -> int:
    """Columns of the widest shard (the slot size of a gathered Y)."""
    n0, n1 = shard_rows(N, world, 0, align)
    return n1 - n0


def gather_shards(y_shard, N: int, group=None):
    """All-gather the ranks' Y shards [M, n1 - n0] into [world, M, shard_width(N)].

    Slot r holds rank r's columns [n0_r, n1_r) of Y, zero-padded on the right to
    the common width; Y[:, n0_r + c] = out[r, :, c]. Uses the process group's
    backend (NCCL over NVLink on GPUs).
    """
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    width = shard_width(N, world)
    M, w = y_shard.shape
    if w != width:
        padded = torch.zeros((M, width), dtype=y_shard.dtype, device=y_shard.device)
        padded[:, :w] = y_shard
        y_shard = padded
    out = torch.empty((world, M, width), dtype=y_shard.dtype, device=y_shard.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, y_shard.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), y_shard.contiguous(), group=group)
    return out
