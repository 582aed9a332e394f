"""Sequence-parallel (Ulysses) attention on CPU gloo ranks.

The all-to-all exchanges of packed_attention_qk_b200.ulysses run over gloo
with 2 and 4 ranks; the attention step inside is the float64 oracle (passed
in by the test), so every rank's output shard must equal the oracle's
attention over the whole packed sequence exactly: the exchanges only move
data ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长", section
"长序列注意力与通信优化": all-to-all from sequence shards to head shards
around attention).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle
from packed_attention_qk_b200 import ulysses

LENS = [300, 0, 513, 1, 210]  # 1024 tokens


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(H, D):
    g = np.random.default_rng(7)
    T = sum(LENS)
    return [g.standard_normal((T, H, D)) for _ in range(3)], np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)


def _oracle_attn(q, k, v, cu, scale):
    o, _ = oracle.varlen_attn(q.contiguous().numpy(), k.contiguous().numpy(), v.contiguous().numpy(), cu.numpy(),
                              scale)
    return torch.from_numpy(o)


def _oracle_prologue(w_q, w_k, pos):
    """The oracle's RMSNorm + RoPE of one head group, written into the send
    buffer's slots (views with their own token strides)."""
    def run(qg, kg, q_out, k_out):
        q_out.copy_(torch.from_numpy(oracle.qk_norm_rope(qg.numpy(), w_q, pos, 1e-6, 10000.0)))
        k_out.copy_(torch.from_numpy(oracle.qk_norm_rope(kg.numpy(), w_k, pos, 1e-6, 10000.0)))
    return run


def _rank_main(rank, world, port, H, D, out, with_prologue=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        (q, k, v), cu = _inputs(H, D)
        T = q.shape[0]
        Tl = T // world
        sl = slice(rank * Tl, (rank + 1) * Tl)
        prologue = None
        if with_prologue:
            g = np.random.default_rng(11)
            w_q, w_k = g.uniform(0.5, 1.5, D), g.uniform(0.5, 1.5, D)
            pos = np.concatenate([np.arange(L) for L in LENS]).astype(np.int32)
            prologue = _oracle_prologue(w_q, w_k, pos[sl])
            qn = oracle.qk_norm_rope(q, w_q, pos, 1e-6, 10000.0)
            kn = oracle.qk_norm_rope(k, w_k, pos, 1e-6, 10000.0)
        o = ulysses.ulysses_attention(torch.from_numpy(q[sl]), torch.from_numpy(k[sl]), torch.from_numpy(v[sl]),
                                      torch.from_numpy(cu), softmax_scale=0.2, attn=_oracle_attn, prologue=prologue,
                                      total_tokens=T)
        if with_prologue:
            ref, _ = oracle.varlen_attn(qn, kn, v, cu, 0.2)
        else:
            ref, _ = oracle.varlen_attn(q, k, v, cu, 0.2)
        out.put((rank, bool(np.array_equal(o.numpy(), ref[sl])), tuple(o.shape)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world, H, with_prologue", [(2, 4, False), (4, 4, False), (4, 8, False), (2, 4, True),
                                                    (4, 8, True)])
def test_shards_equal_the_whole_sequence_attention(world, H, with_prologue):
    # with_prologue: the Q/K norm + RoPE of every head group is written
    # straight into the send buffer and must equal the whole-sequence
    # prologue followed by the whole-sequence attention
    D = 8
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, H, D, out, with_prologue)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=5) for _ in range(world))
    T = sum(LENS)
    assert [g[0] for g in got] == list(range(world))
    assert all(g[1] for g in got), got
    assert all(g[2] == (T // world, H, D) for g in got)


def _bad_rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q = torch.zeros(8, 3, 4, dtype=torch.float64)
        try:
            ulysses.ulysses_attention(q, q, q, torch.tensor([0, 16]), attn=_oracle_attn)
            out.put((rank, "no error"))
        except ValueError as e:
            out.put((rank, str(e)))
    finally:
        dist.destroy_process_group()


def test_heads_not_divisible_by_ranks_is_rejected_before_any_exchange():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bad_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=5) for _ in range(2))
    assert all("divisible" in g[1] for g in got)
