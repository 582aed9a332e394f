"""Property-based pins of the oracle (CPU only, hypothesis): random request
mixes, head counts, head sizes and scales, each checked against a fact that
does not come from the oracle itself.

  * attention = the independent dense padded-and-masked brute force;
  * attention with block skipping and a huge threshold = that brute force;
  * RMSNorm + RoPE preserves every pair's norm of the normalised, weighted
    row and depends on positions only through their differences in dot
    products;
  * e4m3 codes = torch's float8_e4m3fn conversion;
  * the linear layers with their fused epilogues = numpy's matmul followed
    by the residual or SwiGLU, over random request mixes and token strides.
"""

import math

import numpy as np
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import oracle
from tests.bruteforce import padded_masked_attention

lens_st = st.lists(st.integers(min_value=0, max_value=300), min_size=1, max_size=5).filter(lambda l: sum(l) > 0)


@settings(max_examples=25, deadline=None)
@given(lens=lens_st, H=st.integers(1, 3), D=st.sampled_from([4, 8, 16, 32]), scale=st.floats(0.01, 2.0),
       seed=st.integers(0, 2 ** 31 - 1))
def test_attention_equals_bruteforce(lens, H, D, scale, seed):
    g = np.random.default_rng(seed)
    T = sum(lens)
    q, k, v = (g.standard_normal((T, H, D)) for _ in range(3))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, lse = oracle.varlen_attn(q, k, v, cu, scale)
    ob, lb = padded_masked_attention(q, k, v, cu, scale)
    assert np.max(np.abs(o - ob)) <= 1e-11 and np.max(np.abs(lse - lb)) <= 1e-11


@settings(max_examples=15, deadline=None)
@given(lens=lens_st, H=st.integers(1, 2), D=st.sampled_from([8, 16]), seed=st.integers(0, 2 ** 31 - 1))
def test_skip_with_huge_threshold_equals_bruteforce(lens, H, D, seed):
    g = np.random.default_rng(seed)
    T = sum(lens)
    q, k, v = (g.standard_normal((T, H, D)) * 3 for _ in range(3))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, lse, counts = oracle.varlen_attn_skip(q, k, v, cu, 0.3, 1e30, block=(16, 64), tile_rows=64)
    ob, lb = padded_masked_attention(q, k, v, cu, 0.3)
    assert counts == (0, 0)
    assert np.max(np.abs(o - ob)) <= 1e-11 and np.max(np.abs(lse - lb)) <= 1e-11


@settings(max_examples=25, deadline=None)
@given(T=st.integers(1, 40), H=st.integers(1, 3), D=st.sampled_from([4, 8, 64]), style=st.sampled_from([0, 1]),
       base=st.sampled_from([100.0, 10000.0, 500000.0]), seed=st.integers(0, 2 ** 31 - 1))
def test_rope_preserves_pair_norms(T, H, D, style, base, seed):
    g = np.random.default_rng(seed)
    x = g.standard_normal((T, H, D))
    w = g.uniform(0.5, 1.5, D)
    pos = g.integers(0, 200000, T).astype(np.int32)
    y = oracle.qk_norm_rope(x, w, pos, 1e-6, base, style)
    y0 = oracle.qk_norm_rope(x, w, np.zeros(T, np.int32), 1e-6, base, style)
    pairs = [(2 * j, 2 * j + 1) for j in range(D // 2)] if style == 0 else [(j, j + D // 2) for j in range(D // 2)]
    for a, b in pairs:
        np.testing.assert_allclose(y[..., a] ** 2 + y[..., b] ** 2, y0[..., a] ** 2 + y0[..., b] ** 2,
                                   rtol=1e-10, atol=1e-12)


@settings(max_examples=20, deadline=None)
@given(m=st.integers(0, 5000), n=st.integers(0, 5000), shift=st.integers(1, 5000), D=st.sampled_from([4, 16, 64]),
       seed=st.integers(0, 2 ** 31 - 1))
def test_rope_dot_products_depend_on_position_difference(m, n, shift, D, seed):
    g = np.random.default_rng(seed)
    x = g.standard_normal((2, 1, D))
    w = np.ones(D)
    a = oracle.qk_norm_rope(x, w, np.array([m, n], np.int32), 1e-6, 10000.0, 0)
    b = oracle.qk_norm_rope(x, w, np.array([m + shift, n + shift], np.int32), 1e-6, 10000.0, 0)
    assert math.isclose(float(a[0, 0] @ a[1, 0]), float(b[0, 0] @ b[1, 0]), rel_tol=1e-9, abs_tol=1e-9)


@settings(max_examples=30, deadline=None)
@given(st.lists(st.floats(min_value=-448.0, max_value=448.0, width=32), min_size=1, max_size=200))
def test_e4m3_codes_equal_torch(values):
    x = np.array(values, np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_codes(x), ref)


@settings(max_examples=25, deadline=None)
@given(lens=lens_st, K=st.integers(1, 40), N=st.integers(1, 24), pad=st.integers(0, 7),
       seed=st.integers(0, 2 ** 31 - 1))
def test_linear_gated_residual_equals_numpy(lens, K, N, pad, seed):
    # random request mixes (empty ones included) and a token stride of K + pad
    g = np.random.default_rng(seed)
    T = sum(lens)
    wide = g.standard_normal((T, K + pad))
    a = wide[:, :K]
    w, x = g.standard_normal((N, K)), g.standard_normal((T, N))
    gr = g.standard_normal((len(lens), N)).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    seg = np.repeat(np.arange(len(lens)), lens)
    ref = x + gr.astype(np.float64)[seg] * (a @ w.T)
    assert np.max(np.abs(oracle.linear_gated_residual(a, w, x, gr, cu) - ref)) <= 1e-10


@settings(max_examples=25, deadline=None)
@given(T=st.integers(1, 30), K=st.integers(1, 40), F=st.integers(1, 24), seed=st.integers(0, 2 ** 31 - 1))
def test_linear_swiglu_equals_numpy(T, K, F, seed):
    g = np.random.default_rng(seed)
    a, w1 = g.standard_normal((T, K)), g.standard_normal((2 * F, K))
    gate, up = a @ w1[:F].T, a @ w1[F:].T
    ref = gate / (1.0 + np.exp(-gate)) * up
    assert np.max(np.abs(oracle.linear_swiglu(a, w1) - ref) / np.maximum(1.0, np.abs(ref))) <= 1e-12
