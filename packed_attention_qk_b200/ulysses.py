"""Sequence-parallel (Ulysses) packed attention over a process group.

The serving pages shard the ~58k-token joint sequence over 8 GPUs and switch
from sequence shards to head shards around attention with an all-to-all, so
that every GPU attends the whole sequence for H/P heads, exchanging the
shards directly in the layout the attention needs so that no relayout
copies sit around the all-to-alls ("FastH3 在八卡 B300 上实现完整 MP4 生成快于
播放时长", section "长序列注意力与通信优化"; "MiniMax H3 FastH3 real-time serving
with vLLM-Omni", bullet "Long-sequence attention & communication").

Each of the P ranks holds a contiguous shard of T/P tokens of the packed
sequence (shards in rank order) with all H heads. The send buffer is laid
out as [P (destination head group), T/P, 3, H/P, D]: the Q/K prologue
(fused RMSNorm + RoPE) writes each head group's normalised Q and K straight
into their slots through its output strides, and V is copied into its slot
once. One all-to-all moves Q, K and V together; the receive buffer
[P (source token shard), T/P, 3, H/P, D] is the fused [T, 3, H/P, D] layout
the attention kernel reads through its token stride, without a copy. The
attention output [T, H/P, D] is already a [P, T/P, H/P, D] send buffer for
the way back, so the second all-to-all sends it as it is; only the final
[T/P, H, D] interleave of the head groups is a copy. The exchanges are NCCL
collectives on GPUs (gloo on CPU in the tests).
"""

from __future__ import annotations

from typing import Callable


def _attn_default(q, k, v, cu_seqlens, softmax_scale):
    from packed_attention_qk_b200 import pqk
    o, _ = pqk.varlen_attn_fwd(q, k, v, cu_seqlens, softmax_scale=softmax_scale)
    return o


def ulysses_attention(q, k, v, cu_seqlens, *, group=None, softmax_scale: float | None = None,
                      attn: Callable | None = None, prologue: Callable | None = None, total_tokens: int | None = None):
    """q, k, v: this rank's token shard [T/P, H, D] of the packed sequence
    (P = group size; H divisible by P); cu_seqlens: [B+1] offsets of the
    whole packed sequence (0 .. T). Returns this rank's shard of O,
    [T/P, H, D].

    prologue(q_g, k_g, q_out, k_out), when given, writes the normalised and
    rotated Q and K of one head group (views [T/P, H/P, D] of q, k) into
    q_out, k_out (views into the send buffer, with their own token stride),
    e.g. ``pqk.qk_norm_rope(q_g, k_g, w_q, w_k, pos, q_out=q_out, k_out=k_out)``;
    without it q and k are taken as they are. ``attn(q, k, v, cu_seqlens,
    softmax_scale)`` computes the attention of [T, H/P, D] views and returns
    a contiguous [T, H/P, D] output (default: the library's packed varlen
    attention). total_tokens (T), when given, is checked against the shards;
    cu_seqlens is checked only when it is on the host (reading a device
    tensor would synchronise; the attention kernel itself reports bad
    offsets in its status word)."""
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
    if total_tokens is not None and int(total_tokens) != T:
        raise ValueError(f"total_tokens is {total_tokens}, the sharded sequence has {T} tokens")
    if cu_seqlens.device.type == "cpu" and int(cu_seqlens[-1]) != T:
        raise ValueError(f"cu_seqlens ends at {int(cu_seqlens[-1])}, the sharded sequence has {T} tokens")
    attn = attn or _attn_default

    send = torch.empty((P, Tl, 3, Hl, D), dtype=q.dtype, device=q.device)
    for g in range(P):
        heads = slice(g * Hl, (g + 1) * Hl)
        if prologue is not None:
            prologue(q[:, heads], k[:, heads], send[g, :, 0], send[g, :, 1])
        else:
            send[g, :, 0].copy_(q[:, heads])
            send[g, :, 1].copy_(k[:, heads])
    send[:, :, 2].copy_(v.view(Tl, P, Hl, D).transpose(0, 1))
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    fused = recv.view(T, 3, Hl, D)
    o = attn(fused[:, 0], fused[:, 1], fused[:, 2], cu_seqlens, softmax_scale)

    # back: o [T, H/P, D] = [P (destination token shard), T/P, H/P, D] ->
    # [P (source head group), T/P, H/P, D] -> [T/P, H, D]
    back = torch.empty_like(o)
    dist.all_to_all_single(back, o, group=group)
    return back.view(P, Tl, Hl, D).transpose(0, 1).reshape(Tl, H, D)
