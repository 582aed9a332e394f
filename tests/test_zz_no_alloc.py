"""pqk_varlen_attn_fwd_noalloc, the attention entry point for callers that
cannot allocate device memory (for example a plugin handed only its input
and output buffers by a host framework that owns the device heap): it keeps
the tile schedule in a fixed array inside the library instead of a
caller-supplied workspace.

Checked through the C ABI on two calls in a row with different request mixes
(the second call must not see the first call's schedule): the output and the
LSE must equal the workspace entry point's bit for bit (the same kernel on
the same schedule), and both must match the float64 oracle within the
attention tolerances. This file is collected last on purpose; it passes
alone in a fresh process and after the other tests."""

import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import LSE_MAX_ABS, assert_attention, bf16_to_f64, max_abs, to_dev, to_dev_bf16, torch_cuda


@pytest.mark.gpu
def test_no_alloc_entry_matches_workspace_entry_and_oracle_on_two_calls_in_a_row():
    torch = torch_cuda()
    cases = [([1000, 17, 0, 2049], 8, 128), ([200, 312], 4, 64)]
    for lens, H, D in cases:
        w = wl.custom(lens, H, D, seed=sum(lens) + H)
        x = wl.attention_inputs(w)
        q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
        cu = to_dev(x["cu_seqlens"])
        scale = 1.0 / math.sqrt(D)
        o_ref, lse_ref = pqk.varlen_attn_fwd(q, k, v, cu, softmax_scale=scale, want_lse=True)
        o_new, lse_new = pqk.varlen_attn_fwd_noalloc(q, k, v, cu, softmax_scale=scale, want_lse=True)
        torch.cuda.synchronize()
        assert pqk.get_device_status() == 0
        assert torch.equal(o_new.view(torch.int16), o_ref.view(torch.int16)), f"lens {lens}: outputs differ"
        assert torch.equal(lse_new, lse_ref), f"lens {lens}: LSE differs"
        ro, rl = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], scale)
        assert_attention(bf16_to_f64(o_new), ro, f"no-alloc entry vs oracle, lens {lens}")
        assert max_abs(lse_new.cpu().numpy().astype(np.float64).T, rl) <= LSE_MAX_ABS


@pytest.mark.gpu
def test_no_alloc_entry_rejects_a_work_tile_count_beyond_32_bits():
    # 2^31 - 600 tokens x 4096 heads: more 128-row work tiles than the
    # schedule's 32-bit counters hold; rejected on the host, nothing enqueued
    torch_cuda()
    L = pqk.lib()
    A = 0x10000
    T = 2 ** 31 - 600
    rc = L.pqk_varlen_attn_fwd_noalloc(A, A, A, A, None, 4096 * 128, 4096 * 128, 4096 * 128, 4096 * 128, A, 1, T,
                                       4096, 128, 0.088, None)
    assert rc == -1  # PQK_ERR_INVALID_ARG


def test_no_alloc_entry_rejects_more_requests_than_its_array_holds():
    L = pqk.lib()
    A = 0x10000
    rc = L.pqk_varlen_attn_fwd_noalloc(A, A, A, A, None, 1024, 1024, 1024, 1024, A, 4097, 8192, 8, 128, 0.088,
                                       None)
    assert rc == -5  # PQK_ERR_WORKSPACE: B above the fixed schedule capacity
