"""Layout exchange for sequence-parallel callers (plumbing around the hot path).

A video DiT that splits its long token sequence over P ranks holds, per rank, a contiguous
slice of the tokens of every head, token-major [B, T/P, H, d]. The attention of one head
needs all of its tokens, and heads are independent (pooling, ranking and attention never
mix heads), so the usual exchange is one all-to-all to head-parallel [B, T, H/P, d] before
the call and one back after it. With DA2_FLAG_LAYOUT_BTHD and H/P heads in the config,
the head-parallel tensor goes to the library as it is (no transpose). The pages describe
no multi-GPU scheme; this is the plainest one the per-head independence allows.

Both functions call torch.distributed.all_to_all_single on the default (or the given)
process group: NCCL over NVLink on GPUs, gloo on CPU. T and H must be divisible by P.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def seq_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, T/P, H, d] (this rank's tokens, all heads) -> [B, T, H/P, d] (all tokens of this
    rank's H/P heads; rank r gets heads r*H/P .. (r+1)*H/P - 1)."""
    P = dist.get_world_size(group)
    B, Tl, H, d = x.shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    send = x.reshape(B, Tl, P, H // P, d).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)                         # [P (token slice), B, Tl, H/P, d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * Tl, H // P, d)


def heads_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of seq_to_heads: [B, T, H/P, d] -> [B, T/P, H, d]."""
    P = dist.get_world_size(group)
    B, T, Hl, d = y.shape
    if T % P:
        raise ValueError(f"{T} tokens do not split over {P} ranks")
    send = y.reshape(B, P, T // P, Hl, d).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)                         # [P (head group), B, T/P, H/P, d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, T // P, P * Hl, d)
