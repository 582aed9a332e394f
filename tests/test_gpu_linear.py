"""GPU parity of the linear layers with the gated residual or SwiGLU in
the GEMM epilogue (pqk_linear_gated_residual, pqk_linear_swiglu) against
the float64 oracle on the same bf16 inputs, through the C ABI.

Small cases compare every element and span several 128-token tiles, 256-
(or 128-) column tiles and 64-wide K blocks with ragged tails in all three
(T, N and K not multiples of the tile); one case has more tiles than the GPU
has SMs, so every CTA runs several tiles through both tensor-memory
accumulators. The full-size cases (58,048 tokens, hidden 3,072, ffn 8,192)
compare seeded samples of rows, first and last rows included. Tolerances:
the elementwise bounds (the result is one fp32 value rounded to bf16).
"""

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import assert_elementwise, bf16_to_f64, to_dev, to_dev_bf16, torch_cuda

pytestmark = pytest.mark.gpu


def _gated_case(lens, K, N, seed):
    g = np.random.default_rng(seed)
    T = int(sum(lens))
    a = wl.f32_to_bf16_bits(g.standard_normal((T, K)).astype(np.float32))
    w = wl.f32_to_bf16_bits((g.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    x = wl.f32_to_bf16_bits(g.standard_normal((T, N)).astype(np.float32))
    gr = (0.1 * g.standard_normal((len(lens), N))).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return a, w, x, gr, cu


@pytest.mark.parametrize("lens, K, N", [
    ([200, 0, 312, 77], 256, 640),     # 5 token tiles (last ragged), N tail of 128, an empty request
    ([1, 130, 3], 200, 264),           # K = 200: a ragged K block read as zeros past K; N tail of 8
    ([5000], 128, 2048),               # 40 x 8 = 320 tiles > SMs: both accumulators, several tiles per CTA
])
def test_gated_residual_every_element(lens, K, N):
    torch = torch_cuda()
    a, w, x, gr, cu = _gated_case(lens, K, N, seed=K + N)
    out = pqk.linear_gated_residual(to_dev_bf16(a), to_dev_bf16(w), x=to_dev_bf16(x), gate_res=to_dev(gr),
                                    cu_seqlens=to_dev(cu))
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    ref = oracle.linear_gated_residual(a, w, x, gr, cu)
    assert_elementwise(bf16_to_f64(out), ref, f"gated residual {lens} K{K} N{N}")


def test_product_alone_strided_a_and_in_place_residual():
    torch = torch_cuda()
    lens, K, N = [300, 211], 192, 384
    a, w, x, gr, cu = _gated_case(lens, K, N, seed=5)
    T = a.shape[0]
    wide = np.zeros((T, K + 64), np.uint16)
    wide[:, 32:32 + K] = a
    a_view = to_dev_bf16(wide)[:, 32:32 + K]                 # rows K + 64 elements apart
    y = pqk.linear_gated_residual(a_view, to_dev_bf16(w))
    xd = to_dev_bf16(x)
    out = pqk.linear_gated_residual(a_view, to_dev_bf16(w), x=xd, gate_res=to_dev(gr), cu_seqlens=to_dev(cu), out=xd)
    torch.cuda.synchronize()
    assert out.data_ptr() == xd.data_ptr()
    assert_elementwise(bf16_to_f64(y), oracle.linear_gated_residual(a, w), "product alone")
    assert_elementwise(bf16_to_f64(xd), oracle.linear_gated_residual(a, w, x, gr, cu), "in place")


@pytest.mark.parametrize("T, K, F", [(589, 256, 320), (1, 64, 8), (4100, 192, 1024)])
def test_swiglu_every_element(T, K, F):
    torch = torch_cuda()
    g = np.random.default_rng(T + F)
    a = wl.f32_to_bf16_bits(g.standard_normal((T, K)).astype(np.float32))
    w1 = wl.f32_to_bf16_bits((g.standard_normal((2 * F, K)) / np.sqrt(K)).astype(np.float32))
    act = pqk.linear_swiglu(to_dev_bf16(a), to_dev_bf16(w1))
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    assert_elementwise(bf16_to_f64(act), oracle.linear_swiglu(a, w1), f"swiglu T{T} K{K} F{F}")


def test_bitwise_deterministic():
    torch = torch_cuda()
    a, w, x, gr, cu = _gated_case([700, 900], 256, 768, seed=9)
    args = (to_dev_bf16(a), to_dev_bf16(w))
    kw = dict(x=to_dev_bf16(x), gate_res=to_dev(gr), cu_seqlens=to_dev(cu))
    o1 = pqk.linear_gated_residual(*args, **kw)
    o2 = pqk.linear_gated_residual(*args, **kw)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("which", ["o_proj", "w1", "w2"])
def test_full_size_block_layers_sampled_rows(which):
    """The three linear layers of one block at 58,048 tokens (hidden 3,072,
    ffn 8,192), as the bench runs them; 64 sampled rows against the oracle."""
    torch = torch_cuda()
    w = wl.config(3)
    d = wl.linear_inputs(w, which)
    rows = wl.sample_rows(w, per_segment=64)
    a, wt = to_dev_bf16(d["a"]), to_dev_bf16(d["w"])
    if which == "w1":
        out = pqk.linear_swiglu(a, wt)
        ref = oracle.linear_swiglu(d["a"], d["w"], rows=rows)
    else:
        out = pqk.linear_gated_residual(a, wt, x=to_dev_bf16(d["x"]), gate_res=to_dev(d["gate_res"]),
                                        cu_seqlens=to_dev(d["cu_seqlens"]))
        ref = oracle.linear_gated_residual(d["a"], d["w"], d["x"], d["gate_res"], d["cu_seqlens"], rows=rows)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    g = bf16_to_f64(out[torch.from_numpy(rows.astype(np.int64)).cuda()])
    assert_elementwise(g, ref, f"{which} at 58,048 tokens")
