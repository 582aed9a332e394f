"""Failure detection on the GPU without a GPU fault: a bounded wait on a
barrier that nothing completes gives up, records PQK_ERR_TIMEOUT in the
device status word, and the context stays usable afterwards."""

import time

import pytest

from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import assert_attention, bf16_to_f64, to_dev, to_dev_bf16, torch_cuda

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    torch = torch_cuda()
    assert pqk.get_device_status() == 0
    t0 = time.time()
    pqk.selftest_wait_timeout(50_000_000)      # 50 ms
    assert pqk.get_device_status() == -6
    assert time.time() - t0 < 10.0
    assert pqk.get_device_status() == 0
    # the context still runs real work correctly
    from oracle import oracle
    w = wl.config(1)
    x = wl.attention_inputs(w)
    o, _ = pqk.varlen_attn_fwd(to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), to_dev_bf16(x["v"]),
                               to_dev(x["cu_seqlens"]))
    torch.cuda.synchronize()
    ro, _ = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], w.D ** -0.5)
    assert_attention(bf16_to_f64(o), ro, "after timeout")
    assert pqk.get_device_status() == 0
