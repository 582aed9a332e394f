"""Pins for the oracle's linear layers with a fused epilogue (CPU only).

The pages count residual connections and SwiGLU (in place of separate SiLU
and multiply passes) among the DiT operators fused into fewer launches
("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长", section "融合 DiT 算子";
"MiniMax H3 FastH3 real-time serving with vLLM-Omni", bullet "Fused DiT
operators"). Fusing them into the epilogues of the linear layers around them
is a reading: the output projection (or W2) with the gated residual
x' = x + g * (a W^T), and W1 with silu(a W_gate^T) * (a W_up^T).

Pinned by what the weights make exact: the identity, a permutation (which
fixes the orientation of W), a rank-one matrix, the two halves of W1 (which
fixes which half is the SiLU operand), the per-request gate, linearity, and
the product alone against numpy's matmul.
"""

import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import workloads as wl

SILU_1 = 0.7310585786300049  # 1 / (1 + e^-1)


def _rng(seed):
    return np.random.default_rng(seed)


def _silu(v):
    return v / (1.0 + np.exp(-v))


def test_identity_weight_gives_x_plus_gate_times_a():
    g = _rng(1)
    T, K = 7, 16
    a, x = g.standard_normal((T, K)), g.standard_normal((T, K))
    gr = np.float32(g.standard_normal((1, K)))
    out = oracle.linear_gated_residual(a, np.eye(K), x, gr, np.array([0, T]))
    np.testing.assert_allclose(out, x + gr.astype(np.float64) * a, rtol=0, atol=1e-14)


def test_permutation_weight_fixes_the_orientation_of_w():
    # w[n, k] = 1 where k = perm[n]: y[t, n] = a[t, perm[n]]. Reading w as
    # [K, N] would give a[t, perm^-1[n]], which differs for this 3-cycle.
    T, K = 4, 6
    perm = np.array([1, 2, 0, 4, 5, 3])
    w = np.zeros((K, K))
    w[np.arange(K), perm] = 1.0
    a = np.arange(T * K, dtype=np.float64).reshape(T, K)
    y = oracle.linear_gated_residual(a, w)
    assert np.array_equal(y, a[:, perm])
    assert not np.array_equal(y, a[:, np.argsort(perm)])


def test_rank_one_weight_closed_form():
    # w = u v^T (N x K): y[t, n] = u[n] * <a[t], v>
    g = _rng(2)
    T, K, N = 5, 24, 9
    a, u, v = g.standard_normal((T, K)), g.standard_normal(N), g.standard_normal(K)
    y = oracle.linear_gated_residual(a, np.outer(u, v))
    np.testing.assert_allclose(y, np.outer(a @ v, u), rtol=1e-12, atol=1e-12)


def test_non_square_product_equals_numpy_matmul():
    g = _rng(3)
    a, w = g.standard_normal((33, 40)), g.standard_normal((17, 40))
    np.testing.assert_allclose(oracle.linear_gated_residual(a, w), a @ w.T, rtol=1e-12, atol=1e-12)


def test_gate_is_looked_up_per_request_and_zero_gate_keeps_x():
    g = _rng(4)
    lens = [3, 0, 5, 2]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, K, N = int(cu[-1]), 8, 6
    a, w, x = g.standard_normal((T, K)), g.standard_normal((N, K)), g.standard_normal((T, N))
    gr = np.zeros((len(lens), N), np.float32)
    gr[2] = 1.0
    gr[3] = -0.5
    out = oracle.linear_gated_residual(a, w, x, gr, cu)
    y = a @ w.T
    np.testing.assert_array_equal(out[:3], x[:3])                  # request 0: gate 0, x' = x exactly
    np.testing.assert_allclose(out[3:8], x[3:8] + y[3:8], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[8:10], x[8:10] - 0.5 * y[8:10], rtol=1e-12, atol=1e-12)


def test_residual_is_linear_in_a():
    g = _rng(5)
    T, K, N = 6, 12, 10
    a1, a2, w, x = (g.standard_normal(s) for s in ((T, K), (T, K), (N, K), (T, N)))
    gr = np.float32(g.standard_normal((1, N)))
    cu = np.array([0, T])
    f = lambda a: oracle.linear_gated_residual(a, w, x, gr, cu) - x
    np.testing.assert_allclose(f(a1 + a2), f(a1) + f(a2), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f(3.0 * a1), 3.0 * f(a1), rtol=1e-12, atol=1e-12)


def test_strided_a_and_sampled_rows_and_bf16_inputs():
    g = _rng(6)
    T, K, N = 9, 16, 8
    wide = wl.f32_to_bf16_bits(g.standard_normal((T, K + 8)).astype(np.float32))
    a = wide[:, 4:4 + K]                                   # a view with a row stride of K + 8
    w = wl.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32))
    x = wl.f32_to_bf16_bits(g.standard_normal((T, N)).astype(np.float32))
    gr = np.float32(g.standard_normal((1, N)))
    cu = np.array([0, T])
    full = oracle.linear_gated_residual(a, w, x, gr, cu)
    ad, wd, xd = (wl.bf16_bits_to_f64(v) for v in (a, w, x))
    np.testing.assert_allclose(full, xd + gr.astype(np.float64) * (ad @ wd.T), rtol=1e-12, atol=1e-12)
    rows = np.array([8, 0, 5])
    np.testing.assert_array_equal(oracle.linear_gated_residual(a, w, x, gr, cu, rows=rows), full[rows])


def test_gated_residual_rejects_bad_arguments():
    a, w, x = np.ones((4, 8)), np.ones((8, 8)), np.ones((4, 8))
    with pytest.raises(ValueError):
        oracle.linear_gated_residual(a, w, x, np.ones((1, 8), np.float32), np.array([0, 3]))   # cu ends at 3 != T
    with pytest.raises(ValueError):
        oracle.linear_gated_residual(a, w, rows=np.array([4]))                                 # row out of range


def test_swiglu_with_identity_halves():
    g = _rng(7)
    K = 10
    a = g.standard_normal((6, K))
    act = oracle.linear_swiglu(a, np.vstack([np.eye(K), np.eye(K)]))
    np.testing.assert_allclose(act, _silu(a) * a, rtol=1e-14, atol=1e-15)
    ones = oracle.linear_swiglu(np.ones((2, 1)), np.array([[1.0], [1.0]]))
    assert abs(ones[0, 0] - SILU_1) <= 1e-16


def test_swiglu_first_half_is_the_silu_operand():
    # W1 = [P; 2 I]: act = silu(a[:, perm]) * 2 a. With the halves swapped it
    # would be silu(2 a) * a[:, perm].
    K = 4
    perm = np.array([2, 0, 3, 1])
    P = np.zeros((K, K))
    P[np.arange(K), perm] = 1.0
    a = np.array([[1.0, -2.0, 0.5, 3.0]])
    act = oracle.linear_swiglu(a, np.vstack([P, 2.0 * np.eye(K)]))
    np.testing.assert_allclose(act, _silu(a[:, perm]) * 2.0 * a, rtol=1e-14, atol=0)
    assert not np.allclose(act, _silu(2.0 * a) * a[:, perm])


def test_swiglu_zero_gate_half_and_large_gate_limit():
    g = _rng(8)
    K, F = 8, 5
    a = g.standard_normal((3, K))
    wu = g.standard_normal((F, K))
    assert np.array_equal(oracle.linear_swiglu(a, np.vstack([np.zeros((F, K)), wu])), np.zeros((3, F)))
    # a gate of +40 per row: silu(40) = 40 (1 - 4e-18) in float64, act = 40 u
    a1 = np.hstack([np.ones((3, 1)), a])
    wg = np.zeros((F, K + 1))
    wg[:, 0] = 40.0
    wu1 = np.hstack([np.zeros((F, 1)), wu])
    act = oracle.linear_swiglu(a1, np.vstack([wg, wu1]))
    np.testing.assert_allclose(act, 40.0 * (a @ wu.T), rtol=1e-14, atol=1e-14)


def test_swiglu_equals_the_separate_passes():
    # the fused epilogue is the separate SwiGLU pass applied to the two
    # products (numpy matmul for the products)
    g = _rng(9)
    T, K, F = 11, 32, 24
    a, w1 = g.standard_normal((T, K)), g.standard_normal((2 * F, K)) / math.sqrt(K)
    act = oracle.linear_swiglu(a, w1)
    _, _, ref = oracle.modulate_swiglu(np.ones((T, 8)), np.zeros((1, 8), np.float32), np.zeros((1, 8), np.float32),
                                       np.zeros((1, 8), np.float32), np.array([0, T]), gate=a @ w1[:F].T,
                                       up=a @ w1[F:].T)
    np.testing.assert_allclose(act, ref, rtol=1e-12, atol=1e-13)
    rows = np.array([10, 3])
    np.testing.assert_array_equal(oracle.linear_swiglu(a, w1, rows=rows), act[rows])
