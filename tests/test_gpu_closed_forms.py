"""GPU results against closed forms (no oracle): the degenerate cases of the
three operations, where the exact answer is known in advance.

  * attention with Q = 0: every key has the same score, so each row's output
    is the mean of its request's V rows and lse = ln L;
  * one-token requests: O = V exactly (the single probability is 1) and
    lse = the single score;
  * RMSNorm + RoPE at position 0 with a constant row c: y = w c / sqrt(c^2 + eps);
  * modulation with norm NONE and zero shift, scale and gate: h = x and
    x' = x exactly.
"""

import math

import numpy as np
import pytest

from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import ATTN_MAX_ABS, LSE_MAX_ABS, bf16_to_f64, max_abs, to_dev, to_dev_bf16, torch_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128])
def test_zero_queries_give_the_mean_of_v(D):
    torch = torch_cuda()
    lens = [1, 200, 0, 1000, 129]
    w = wl.custom(lens, 3, D, seed=71)
    x = wl.attention_inputs(w)
    q = torch.zeros((w.T, w.H, D), dtype=torch.bfloat16, device="cuda")
    o, lse = pqk.varlen_attn_fwd(q, to_dev_bf16(x["k"]), to_dev_bf16(x["v"]), to_dev(x["cu_seqlens"]),
                                 want_lse=True)
    torch.cuda.synchronize()
    v = wl.bf16_bits_to_f64(x["v"])
    cu = x["cu_seqlens"]
    g, gl = bf16_to_f64(o), lse.cpu().numpy().astype(np.float64).T
    for i in range(len(lens)):
        lo, hi = int(cu[i]), int(cu[i + 1])
        if hi == lo:
            continue
        assert max_abs(g[lo:hi], np.broadcast_to(v[lo:hi].mean(axis=0), g[lo:hi].shape)) <= ATTN_MAX_ABS
        assert np.max(np.abs(gl[lo:hi] - math.log(hi - lo))) <= LSE_MAX_ABS


def test_one_token_requests_return_v_exactly():
    torch = torch_cuda()
    n, H, D = 700, 4, 128
    w = wl.custom([1] * n, H, D, seed=72)
    x = wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(D)
    v = to_dev_bf16(x["v"])
    o, lse = pqk.varlen_attn_fwd(to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), v, to_dev(x["cu_seqlens"]),
                                 softmax_scale=scale, want_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), v.view(torch.int16))
    q, k = wl.bf16_bits_to_f64(x["q"]), wl.bf16_bits_to_f64(x["k"])
    s = scale * np.einsum("thd,thd->th", q, k)
    assert np.max(np.abs(lse.cpu().numpy().astype(np.float64).T - s)) <= LSE_MAX_ABS


def test_norm_rope_of_constant_rows_at_position_zero():
    torch = torch_cuda()
    T, H, D, eps = 40, 4, 128, 1e-6
    c = np.linspace(-3.0, 3.0, T * H).reshape(T, H, 1)
    xq = wl.f32_to_bf16_bits(np.broadcast_to(c, (T, H, D)).astype(np.float32))
    wq = wl.f32_to_bf16_bits(np.linspace(0.5, 1.5, D).astype(np.float32))
    q, k = to_dev_bf16(xq), to_dev_bf16(xq)
    wd = to_dev_bf16(wq)
    pqk.qk_norm_rope(q, k, wd, wd, torch.zeros(T, dtype=torch.int32, device="cuda"), eps=eps)
    torch.cuda.synchronize()
    cb = wl.bf16_bits_to_f64(xq)[..., :1]
    expect = wl.bf16_bits_to_f64(wq)[None, None, :] * cb / np.sqrt(cb ** 2 + eps)
    g = bf16_to_f64(q)
    assert np.max(np.abs(g - expect) / np.maximum(1.0, np.abs(expect))) <= 1e-2
    assert torch.equal(q.view(torch.int16), k.view(torch.int16))


def test_modulation_none_with_zero_vectors_is_the_identity():
    torch = torch_cuda()
    w = wl.custom([300, 0, 77], 4, 64, seed=73)
    e = wl.epilogue_inputs(w, with_branch=True)
    x = to_dev_bf16(e["x"])
    z = torch.zeros((w.B, w.C), dtype=torch.float32, device="cuda")
    xo, h, _ = pqk.modulate_swiglu(x, z, z, to_dev(w.cu_seqlens()), gate_res=z, branch=to_dev_bf16(e["branch"]),
                                   norm_type=pqk.NORM_NONE, x_out=torch.empty_like(x))
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int16), x.view(torch.int16))
    assert torch.equal(xo.view(torch.int16), x.view(torch.int16))
