"""Sequence-parallel (Ulysses) packed attention over a process group.

The serving pages shard the ~58k-token joint sequence over 8 GPUs and switch
from sequence shards to head shards around attention with an all-to-all, so
that every GPU attends the whole sequence for H/P heads ("FastH3 在八卡 B300
上实现完整 MP4 生成快于播放时长", section "长序列注意力与通信优化"; "MiniMax H3
FastH3 real-time serving with vLLM-Omni", bullet "Long-sequence attention &
communication").

Each of the P ranks holds a contiguous shard of T/P tokens of the packed
sequence (shards in rank order) with all H heads. One all-to-all moves Q, K
and V together to "all T tokens, this rank's H/P heads" in a fused
[T, 3, H/P, D] layout, which the attention kernel reads through its token
stride without a copy; the attention runs over every request of the packed
sequence; a second all-to-all returns O to the token shards. The exchanges
are NCCL collectives on GPUs (gloo on CPU in the tests); the only data
movement outside the collectives is one permute of the send buffer each way.
"""

from __future__ import annotations

from typing import Callable


def _attn_default(q, k, v, cu_seqlens, softmax_scale):
    from packed_attention_qk_b200 import pqk
    o, _ = pqk.varlen_attn_fwd(q, k, v, cu_seqlens, softmax_scale=softmax_scale)
    return o


def ulysses_attention(q, k, v, cu_seqlens, *, group=None, softmax_scale: float | None = None,
                      attn: Callable | None = None):
    """q, k, v: this rank's token shard [T/P, H, D] of the packed sequence
    (P = group size; T and H divisible by P); cu_seqlens: [B+1] offsets of
    the whole packed sequence (0 .. T). Returns this rank's shard of O,
    [T/P, H, D]. ``attn(q, k, v, cu_seqlens, softmax_scale)`` computes the
    attention of [T, H/P, D] views (default: the library's packed varlen
    attention)."""
    import torch
    import torch.distributed as dist

    P = dist.get_world_size(group)
    Tl, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v shards must have the same shape")
    if H % P:
        raise ValueError(f"heads ({H}) must be divisible by the group size ({P})")
    Hl = H // P
    T = Tl * P
    if int(cu_seqlens[-1]) != T:
        raise ValueError(f"cu_seqlens ends at {int(cu_seqlens[-1])}, the sharded sequence has {T} tokens")
    attn = attn or _attn_default

    # send buffer [P (destination head group), T/P, 3, H/P, D]; receive buffer
    # [P (source token shard), T/P, 3, H/P, D] = [T, 3, H/P, D]
    qkv = torch.stack((q, k, v), dim=1).view(Tl, 3, P, Hl, D)
    send = qkv.permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    fused = recv.view(T, 3, Hl, D)
    o = attn(fused[:, 0], fused[:, 1], fused[:, 2], cu_seqlens, softmax_scale)

    # back: [P (destination token shard), T/P, H/P, D] -> [P (source head
    # group), T/P, H/P, D] -> [T/P, H, D]
    o = o.contiguous()
    back = torch.empty_like(o)
    dist.all_to_all_single(back, o, group=group)
    return back.view(P, Tl, Hl, D).permute(1, 0, 2, 3).reshape(Tl, H, D)
