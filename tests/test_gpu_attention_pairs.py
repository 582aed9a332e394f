"""The attention on CTA pairs (pqk_set_attn_cta_pairs): two SMs share each
512-row work tile and one thread issues the pair's tcgen05 cta_group::2
products. Its results must be bit-identical to the one-SM kernel's (each
row's products, softmax and rounding are the same; only which SM computes
what changes), on ragged and empty requests, tails of every size modulo 512
and 128, many short requests and the full-size joint sequence, and it must
match the float64 oracle on its own; a pipeline timeout must be reported,
drained and recovered from as in the one-SM kernel."""

import contextlib
import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import (LSE_MAX_ABS, assert_attention, bf16_to_f64, max_abs, to_dev, to_dev_bf16,
                             torch_cuda)

pytestmark = pytest.mark.gpu
TIMEOUT = -6


@contextlib.contextmanager
def cta_pairs(enable=True):
    pqk.set_attn_cta_pairs(enable)
    try:
        yield
    finally:
        pqk.set_attn_cta_pairs(False)


def _both(x):
    torch = torch_cuda()
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    cu = to_dev(x["cu_seqlens"])
    o1, l1 = pqk.varlen_attn_fwd(q, k, v, cu, want_lse=True)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    with cta_pairs():
        o2, l2 = pqk.varlen_attn_fwd(q, k, v, cu, want_lse=True)
        torch.cuda.synchronize()
        assert pqk.get_device_status() == 0
    return (o1, l1), (o2, l2)


@pytest.mark.parametrize("lens", [[1], [128], [255], [256], [257], [511], [512], [513], [300, 0, 513, 1],
                                  [0, 0, 700], [384, 17, 2, 640, 1025], [4096, 1000, 0, 129]])
def test_pairs_are_bitwise_the_one_sm_kernel(lens):
    torch = torch_cuda()
    w = wl.custom(lens, 3, 128, seed=81)
    (o1, l1), (o2, l2) = _both(wl.attention_inputs(w))
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)), f"{lens}: O differs"
    assert torch.equal(l1, l2), f"{lens}: LSE differs"


def test_pairs_many_short_requests_bitwise():
    torch = torch_cuda()
    g = np.random.default_rng(82)
    lens = g.integers(0, 700, 300).tolist()
    w = wl.custom(lens, 2, 128, seed=82)
    (o1, l1), (o2, l2) = _both(wl.attention_inputs(w))
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_pairs_against_the_oracle():
    w = wl.custom([700, 1, 1300, 0, 257], 4, 128, seed=83)
    x = wl.attention_inputs(w)
    torch = torch_cuda()
    with cta_pairs():
        o, lse = pqk.varlen_attn_fwd(to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), to_dev_bf16(x["v"]),
                                     to_dev(x["cu_seqlens"]), want_lse=True)
        torch.cuda.synchronize()
        assert pqk.get_device_status() == 0
    ro, rl = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], 1.0 / math.sqrt(128))
    assert_attention(bf16_to_f64(o), ro, "CTA pairs")
    assert max_abs(lse.cpu().numpy().astype(np.float64).T, rl) <= LSE_MAX_ABS


def test_pairs_joint_sequence_58048_bitwise_and_sampled():
    torch = torch_cuda()
    w = wl.config(3)
    x = wl.attention_inputs(w)
    (o1, l1), (o2, l2) = _both(x)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)
    rows = wl.sample_rows(w, 64)
    ro, rl = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], 1.0 / math.sqrt(w.D), rows=rows)
    assert_attention(bf16_to_f64(o2)[rows], ro, "CTA pairs, 58,048 tokens")
    assert max_abs(l2.cpu().numpy().astype(np.float64).T[rows], rl) <= LSE_MAX_ABS


def test_pairs_pipeline_timeout_is_reported_drained_and_recovered():
    torch = torch_cuda()
    w = wl.custom([4096, 1000, 0, 129], 8, 128, seed=84)
    x = wl.attention_inputs(w)
    T, H, D = w.T, w.H, w.D
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    cu = to_dev(x["cu_seqlens"])
    o_full = torch.full((T + 16, H * D + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    o = o_full[8:8 + T, :H * D].view(T, H, D)
    fired = False
    with cta_pairs():
        pqk.set_wait_timeout_ns(1000)
        try:
            for _ in range(3):
                pqk.varlen_attn_fwd(q, k, v, cu, o=o)
                st = pqk.get_device_status()
                assert st in (0, TIMEOUT), f"unexpected status {st}"
                if st == TIMEOUT:
                    fired = True
                    break
        finally:
            pqk.set_wait_timeout_ns(0)
        assert fired
        guard = torch.cat([o_full[:8].flatten(), o_full[8 + T:].flatten(), o_full[8:8 + T, H * D:].flatten()])
        assert bool((guard == 7.0).all()), "written outside O"
        o2, lse2 = pqk.varlen_attn_fwd(q, k, v, cu, want_lse=True)
        torch.cuda.synchronize()
        assert pqk.get_device_status() == 0
    rows = wl.sample_rows(w, 64)
    ro, rl = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], 1.0 / math.sqrt(D), rows=rows)
    assert_attention(bf16_to_f64(o2)[rows], ro, "CTA pairs after a timed-out call")
    assert max_abs(lse2.cpu().numpy().astype(np.float64).T[rows], rl) <= LSE_MAX_ABS


def test_pairs_no_alloc_entry_bitwise():
    # the no-allocation entry keeps its schedule (512-row work tiles on pairs)
    # in the library's own array: same results as the one-SM workspace entry
    torch = torch_cuda()
    w = wl.custom([1000, 17, 0, 2049], 8, 128, seed=85)
    x = wl.attention_inputs(w)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    cu = to_dev(x["cu_seqlens"])
    o1, l1 = pqk.varlen_attn_fwd(q, k, v, cu, want_lse=True)
    with cta_pairs():
        o2, l2 = pqk.varlen_attn_fwd_noalloc(q, k, v, cu, want_lse=True)
        torch.cuda.synchronize()
        assert pqk.get_device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)
