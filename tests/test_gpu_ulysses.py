"""The Ulysses exchange on a GPU: a one-rank NCCL group (the only size one
GPU allows), so both all-to-alls are local copies and the attention runs on
the fused [T, 3, H, D] receive buffer through its token stride. The result
must equal the library's attention on contiguous inputs bit for bit, and
both must match the float64 oracle on the unsharded inputs within the
attention tolerances. Exchanges across several GPUs are covered by the gloo
tests on CPU."""

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
        o = ulysses.ulysses_attention(q, k, v, cu, softmax_scale=0.1)
        ref, _ = pqk.varlen_attn_fwd(q, k, v, cu, softmax_scale=0.1)
        torch.cuda.synchronize()
        assert pqk.get_device_status() == 0
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
        ro, _ = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], 0.1)
        assert_attention(bf16_to_f64(o), ro, "one-rank Ulysses vs oracle")
    finally:
        dist.destroy_process_group()
