"""The Ulysses exchange on a GPU: a one-rank NCCL group (the only size one
GPU allows), so both all-to-alls are local copies and the attention runs on
the fused [T, 3, H, D] receive buffer through its token stride. The result
must equal the library's attention on contiguous inputs bit for bit, and
both must match the float64 oracle on the unsharded inputs within the
attention tolerances; with the Q/K prologue writing straight into the send
buffer, the result must equal the prologue run out of place followed by the
attention, bit for bit. Exchanges across several GPUs are covered by the
gloo tests on CPU."""

import os
import socket

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk, ulysses
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import assert_attention, bf16_to_f64, to_dev, to_dev_bf16, torch_cuda

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_group_equals_plain_attention():
    torch = torch_cuda()
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        w = wl.custom([300, 0, 513, 1, 210], 4, 128, seed=3)
        x = wl.attention_inputs(w)
        q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
        cu = to_dev(x["cu_seqlens"])
        o = ulysses.ulysses_attention(q, k, v, cu, softmax_scale=0.1, total_tokens=w.T)
        ref, _ = pqk.varlen_attn_fwd(q, k, v, cu, softmax_scale=0.1)
        torch.cuda.synchronize()
        assert pqk.get_device_status() == 0
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
        ro, _ = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], 0.1)
        assert_attention(bf16_to_f64(o), ro, "one-rank Ulysses vs oracle")

        # the prologue writes the normalised, rotated Q and K into the send buffer
        p = wl.prologue_inputs(w)
        wq, wk, pos = to_dev_bf16(p["w_q"]), to_dev_bf16(p["w_k"]), to_dev(p["pos"])
        prologue = lambda qg, kg, qo, ko: pqk.qk_norm_rope(qg, kg, wq, wk, pos, eps=w.eps, rope_base=w.rope_base,
                                                           q_out=qo, k_out=ko)
        o2 = ulysses.ulysses_attention(q, k, v, cu, softmax_scale=0.1, prologue=prologue, total_tokens=w.T)
        qn, kn = torch.empty_like(q), torch.empty_like(k)
        pqk.qk_norm_rope(q, k, wq, wk, pos, eps=w.eps, rope_base=w.rope_base, q_out=qn, k_out=kn)
        ref2, _ = pqk.varlen_attn_fwd(qn, kn, v, cu, softmax_scale=0.1)
        torch.cuda.synchronize()
        assert pqk.get_device_status() == 0
        assert torch.equal(o2.view(torch.int16), ref2.view(torch.int16))
        rq = oracle.qk_norm_rope(x["q"], p["w_q"], p["pos"], w.eps, w.rope_base)
        rk = oracle.qk_norm_rope(x["k"], p["w_k"], p["pos"], w.eps, w.rope_base)
        ro2, _ = oracle.varlen_attn(rq, rk, wl.bf16_bits_to_f64(x["v"]), x["cu_seqlens"], 0.1)
        assert_attention(bf16_to_f64(o2), ro2, "one-rank Ulysses with the prologue vs oracle")
    finally:
        dist.destroy_process_group()
