"""Tensor-parallel (column / N-split) W4A4 linear: each rank holds a contiguous range of the folded
weight's output rows and computes those output columns for the full batch; the shards' outputs are
all-gathered along N.

Why this split: every Hadamard and MX block covers 32 consecutive input channels of ONE output row
("MACaQ ...", Abstract: the transforms are local to each layer and folded into its weights), so
output rows shard with no exchange of transforms or scales, and the activations' transform and
quantisation are the same on every rank (each rank quantises its replica of x).  The only
collective is the all-gather of the bf16 outputs (NCCL over NVLink on GPUs; gloo in the CPU tests).

Shards are whole 128-row blocks: the E8M0 scales of a 128-row block are one contiguous run of
bytes in the MMA tile layout (include/macaq.h), so a shard's codes and scales are plain slices of
the folded buffers.  Ranks get ceil(blocks / world) or floor(blocks / world) blocks, in rank
order; the last shard may end with a partial block.
"""
from __future__ import annotations

import torch

BLOCK_ROWS = 128


def shard_range(N: int, world: int, rank: int) -> tuple[int, int]:
    """Output rows [n0, n1) of `rank`: whole 128-row blocks, the first (blocks % world) ranks one
    block more, the last shard ending at N."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    blocks = (N + BLOCK_ROWS - 1) // BLOCK_ROWS
    base, extra = divmod(blocks, world)
    b0 = rank * base + min(rank, extra)
    b1 = b0 + base + (1 if rank < extra else 0)
    return min(b0 * BLOCK_ROWS, N), min(b1 * BLOCK_ROWS, N)


def scale_block_bytes(K: int) -> int:
    """Bytes of the E8M0 scales of one 128-row block in the MMA tile layout."""
    return BLOCK_ROWS * 8 * ((K + 255) // 256)


def shard_folded_weights(Wq: torch.Tensor, Ws: torch.Tensor, N: int, K: int, world: int, rank: int):
    """This rank's slice of folded weights (codes [N, K/2], scales in the MMA tile layout):
    (codes [n1 - n0, K/2], scales, n1 - n0).  Views, no copies."""
    n0, n1 = shard_range(N, world, rank)
    sb = scale_block_bytes(K)
    b0, b1 = n0 // BLOCK_ROWS, (n1 + BLOCK_ROWS - 1) // BLOCK_ROWS
    return Wq[n0:n1], Ws[b0 * sb:b1 * sb], n1 - n0


def gather_columns(y_shard: torch.Tensor, N: int, group=None) -> torch.Tensor:
    """All-gather every rank's output columns [M, n1 - n0] into y [M, N] (rank order = column order)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if world == 1:
        return y_shard
    M = y_shard.shape[0]
    widths = [shard_range(N, world, r)[1] - shard_range(N, world, r)[0] for r in range(world)]
    wmax = max(widths)
    send = y_shard
    if y_shard.shape[1] < wmax:  # equal-sized messages: pad the narrower shards
        send = torch.zeros(M, wmax, dtype=y_shard.dtype, device=y_shard.device)
        send[:, :y_shard.shape[1]] = y_shard
    parts = [torch.empty(M, wmax, dtype=y_shard.dtype, device=y_shard.device) for _ in range(world)]
    dist.all_gather(parts, send.contiguous(), group=group)
    return torch.cat([p[:, :w] for p, w in zip(parts, widths)], dim=1)


def tp_w4a4_linear(x: torch.Tensor, act_mult: torch.Tensor, Wq_shard: torch.Tensor, Ws_shard: torch.Tensor,
                   N: int, group=None, workspace=None, stream=None) -> torch.Tensor:
    """y = x W^T over the ranks of `group`: this rank's W4A4 linear on its weight shard (from
    shard_folded_weights), then the all-gather of the output columns."""
    from . import macaq_w4a4_linear
    if Wq_shard.shape[0] == 0:  # more ranks than 128-row blocks: nothing to compute here
        y_shard = torch.empty(x.shape[0], 0, dtype=torch.bfloat16, device=x.device)
    else:
        y_shard = macaq_w4a4_linear(x, act_mult, Wq_shard, Ws_shard, Wq_shard.shape[0], workspace=workspace,
                                    stream=stream)
    return gather_columns(y_shard, N, group)
