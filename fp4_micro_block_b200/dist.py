"""Host-side helpers for running the quantizer on several GPUs (one process per GPU).

Rows (tokens) are independent, so the path shards by rows and needs no data
exchange.  The one optional collective is for an NVFP4 tensor scale shared by
all ranks: s_t = amax/2688 is monotone in amax (an IEEE division by a positive
constant), so the MAX over ranks of the local s_t equals the s_t of the global
amax exactly; one all-reduce of one float gives it, after which every rank
quantizes with FP4Q_TSCALE_STATIC.

fp4_all_gather is the FP4-compressed exchange of the FP4Quant abstract (model-
parallel communication compressed to FP4): each rank quantizes its block of
activations (dual scale after a block Hadamard rotation), one all-gather moves
the packed payloads (0.59 bytes per element instead of 2), and every rank
dequantizes and rotates back all blocks.
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


# --------------------------------------------------------------------------- FP4-compressed all-gather

def _up16(n: int) -> int:
    return (n + 15) // 16 * 16


def payload_bytes(m: int, K: int) -> int:
    """Bytes of one rank's payload for an [m, K] block: packed codes [m, K/2],
    E4M3 micro-scales [m, K/16] and FP32 group scales [m, K/128], each section
    starting on a 16-byte boundary."""
    if K % 128:
        raise ValueError("the dual format needs K % 128 == 0")
    return _up16(m * K // 2) + _up16(m * K // 16) + _up16(m * (K // 128) * 4)


def payload_views(buf: torch.Tensor, m: int, K: int):
    """(codes [m, K/2] u8, scales [m, K/16] u8, group scales [m, K/128] f32) views
    into a uint8 payload buffer of payload_bytes(m, K) bytes."""
    if buf.dtype != torch.uint8 or buf.numel() < payload_bytes(m, K):
        raise ValueError("payload buffer too small")
    o1 = _up16(m * K // 2)
    o2 = o1 + _up16(m * K // 16)
    codes = buf[: m * K // 2].view(m, K // 2)
    scales = buf[o1: o1 + m * K // 16].view(m, K // 16)
    g = buf[o2: o2 + m * (K // 128) * 4].view(torch.float32).view(m, K // 128)
    return codes, scales, g


class KernelCodec:
    """Quantize / dequantize of a block through the library's kernels: dual
    scale after a block Hadamard rotation of size `had_size`, and back."""

    def __init__(self, had_size: int = 512):
        self.had_size = had_size

    def quantize(self, x, codes, scales, g):
        import fp4_micro_block_b200 as fq
        fq.fp4q_hadamard_quantize(x, self.had_size, fq.FP4Q_NVFP4_DUAL, codes, scales, g)

    def dequantize(self, codes, scales, g, y):
        import fp4_micro_block_b200 as fq
        fq.fp4q_dequantize(fq.FP4Q_NVFP4_DUAL, codes, scales, g, y.shape[0], y.shape[1], y,
                           fq.FP4Q_SCALES_LINEAR, self.had_size)


def fp4_all_gather(x: torch.Tensor, group=None, codec=None) -> torch.Tensor:
    """All-gather of bf16 activations [m, K] (the same m on every rank) in FP4:
    returns the [world * m, K] bf16 round trip of every rank's block, in rank
    order.  One collective carries each rank's packed payload; the receiver
    dequantizes the blocks one by one.  `codec` defaults to the kernels
    (KernelCodec); any object with the same quantize / dequantize methods
    works."""
    codec = KernelCodec() if codec is None else codec
    world = dist.get_world_size(group)
    m, K = x.shape
    nb = payload_bytes(m, K)
    send = torch.empty(nb, dtype=torch.uint8, device=x.device)  # section padding is never read
    codec.quantize(x, *payload_views(send, m, K))
    recv = torch.empty(world * nb, dtype=torch.uint8, device=x.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    out = torch.empty((world * m, K), dtype=torch.bfloat16, device=x.device)
    for r in range(world):
        codec.dequantize(*payload_views(recv[r * nb:(r + 1) * nb], m, K), out[r * m:(r + 1) * m])
    return out
