"""Host-side helpers for running the quantizer on several GPUs (one process per GPU).

Rows (tokens) are independent, so the path shards by rows and needs no data
exchange.  The one optional collective is for an NVFP4 tensor scale shared by
all ranks: s_t = amax/2688 is monotone in amax (an IEEE division by a positive
constant), so the MAX over ranks of the local s_t equals the s_t of the global
amax exactly; one all-reduce of one float gives it, after which every rank
quantizes with FP4Q_TSCALE_STATIC.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

ROW_ALIGN = 128  # a tile of the 128x4 scale layout never straddles two ranks


def row_range(M: int, rank: int, world: int, align: int = ROW_ALIGN) -> tuple[int, int]:
    """Contiguous rows [start, stop) of rank `rank`; shard boundaries are multiples
    of `align` (the last shard takes the remainder)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    blocks = (M + align - 1) // align
    per, extra = divmod(blocks, world)
    b0 = rank * per + min(rank, extra)
    b1 = b0 + per + (1 if rank < extra else 0)
    return min(M, b0 * align), min(M, b1 * align)


def global_tensor_scale(local_scale: torch.Tensor, group=None) -> torch.Tensor:
    """In place: MAX all-reduce of a 1-float tensor scale (NCCL for CUDA tensors,
    gloo for CPU tensors)."""
    dist.all_reduce(local_scale, op=dist.ReduceOp.MAX, group=group)
    return local_scale
