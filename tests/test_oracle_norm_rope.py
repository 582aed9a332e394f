"""Pins for the oracle's fused Q/K RMSNorm + RoPE (CPU only).

The pages name the operation ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长",
section "融合 DiT 算子": Q/K normalisation merged with RoPE) but print no
example, so the oracle is pinned by closed forms and by properties any
correct RMSNorm + rotary embedding has: unit RMS before the weight, rotation
preserves each pair's norm, position 0 is the identity, dot products depend
only on the position difference, and rotations compose.
"""

import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import workloads as wl

IL, HALF = oracle.ROPE_INTERLEAVED, oracle.ROPE_HALF


def _pairs(D, style):
    if style == IL:
        return [(2 * j, 2 * j + 1) for j in range(D // 2)]
    return [(j, j + D // 2) for j in range(D // 2)]


@pytest.mark.parametrize("style", [IL, HALF])
def test_unit_rms_before_weight(style):
    # with pos = 0 the output is the normalised row times w, and
    # mean((y / w)^2) = ms / (ms + eps) exactly
    g = np.random.default_rng(0)
    T, H, D, eps = 9, 3, 64, 0.01
    x = g.standard_normal((T, H, D)) * 0.3
    w = g.uniform(0.5, 1.5, D)
    y = oracle.qk_norm_rope(x, w, np.zeros(T, np.int32), eps, 10000.0, style)
    ms = (x ** 2).mean(axis=-1)
    np.testing.assert_allclose(((y / w) ** 2).mean(axis=-1), ms / (ms + eps), rtol=1e-13)


def test_constant_row_closed_form():
    # x = c everywhere: y_d = w_d c / sqrt(c^2 + eps); eps = 1, c = 1 gives 1/sqrt(2)
    T, H, D = 1, 1, 8
    x = np.ones((T, H, D))
    w = np.arange(1, D + 1, dtype=np.float64)
    y = oracle.qk_norm_rope(x, w, np.zeros(T, np.int32), 1.0, 10000.0, IL)
    np.testing.assert_allclose(y[0, 0], w / math.sqrt(2.0), rtol=1e-15)


def test_rotation_sign_and_frequency_closed_form():
    # D = 4, base 10000: theta_0 = 1, theta_1 = 10000^(-1/2) = 0.01.
    # Unit pairs rotated counter-clockwise: (1, 0) -> (cos phi, sin phi).
    D = 4
    w = np.ones(D)
    x = np.zeros((1, 1, D))
    x[0, 0, 0] = 1.0          # interleaved pair 0 = (x0, x1)
    x[0, 0, 2] = 1.0          # interleaved pair 1 = (x2, x3)
    eps = 0.0
    for pos in (1, 100, 186488):
        y = oracle.qk_norm_rope(x, w, np.array([pos], np.int32), eps, 10000.0, IL)[0, 0]
        r = math.sqrt(2.0)     # RMS of (1, 0, 1, 0) is 1/sqrt(2)
        np.testing.assert_allclose(y, [r * math.cos(pos), r * math.sin(pos),
                                       r * math.cos(0.01 * pos), r * math.sin(0.01 * pos)], atol=1e-12)


def test_half_pairing_closed_form():
    # HALF pairs (j, j + D/2): a unit at index 0 rotates into index D/2
    D = 4
    x = np.zeros((1, 1, D))
    x[0, 0, 0] = 1.0
    y = oracle.qk_norm_rope(x, np.ones(D), np.array([3], np.int32), 0.0, 10000.0, HALF)[0, 0]
    np.testing.assert_allclose(y, [2 * math.cos(3), 0.0, 2 * math.sin(3), 0.0], atol=1e-14)


@pytest.mark.parametrize("style", [IL, HALF])
def test_rotation_preserves_pair_norms_and_pos0_is_identity(style):
    g = np.random.default_rng(1)
    T, H, D = 16, 2, 128
    x = wl.f32_to_bf16_bits(g.standard_normal((T, H, D)).astype(np.float32))
    w = wl.f32_to_bf16_bits(g.uniform(0.5, 1.5, D).astype(np.float32))
    pos = g.integers(0, 186489, T).astype(np.int32)
    y = oracle.qk_norm_rope(x, w, pos, 1e-6, 10000.0, style)
    y0 = oracle.qk_norm_rope(x, w, np.zeros(T, np.int32), 1e-6, 10000.0, style)
    xf, wf = wl.bf16_bits_to_f64(x), wl.bf16_bits_to_f64(w)
    n = xf / np.sqrt((xf ** 2).mean(-1, keepdims=True) + 1e-6) * wf
    np.testing.assert_allclose(y0, n, atol=1e-14)
    for a, b in _pairs(D, style):
        np.testing.assert_allclose(y[..., a] ** 2 + y[..., b] ** 2, y0[..., a] ** 2 + y0[..., b] ** 2,
                                   rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("style", [IL, HALF])
def test_dot_product_depends_only_on_position_difference(style):
    g = np.random.default_rng(2)
    H, D = 1, 64
    q = g.standard_normal((1, H, D))
    k = g.standard_normal((1, H, D))
    w = np.ones(D)
    for m, n in [(5, 3), (1000, 17), (55295, 512)]:
        qm = oracle.qk_norm_rope(q, w, np.array([m], np.int32), 1e-6, 10000.0, style)
        kn = oracle.qk_norm_rope(k, w, np.array([n], np.int32), 1e-6, 10000.0, style)
        qd = oracle.qk_norm_rope(q, w, np.array([m - n], np.int32), 1e-6, 10000.0, style)
        k0 = oracle.qk_norm_rope(k, w, np.array([0], np.int32), 1e-6, 10000.0, style)
        assert abs(np.sum(qm * kn) - np.sum(qd * k0)) <= 1e-10


@pytest.mark.parametrize("style", [IL, HALF])
def test_rotations_compose(style):
    # with w = 1 and eps = 0 the normalised row has RMS 1, so a second pass
    # only rotates: R(b) R(a) x = R(a + b) x
    g = np.random.default_rng(3)
    T, H, D = 6, 2, 32
    x = g.standard_normal((T, H, D))
    w = np.ones(D)
    a = g.integers(0, 5000, T).astype(np.int32)
    b = g.integers(0, 5000, T).astype(np.int32)
    y1 = oracle.qk_norm_rope(x, w, a, 0.0, 10000.0, style)
    y2 = oracle.qk_norm_rope(y1, w, b, 0.0, 10000.0, style)
    y3 = oracle.qk_norm_rope(x, w, a + b, 0.0, 10000.0, style)
    np.testing.assert_allclose(y2, y3, atol=1e-11)


def test_strided_token_view_of_a_fused_buffer():
    # q as the first H*D columns of a [T, 3*H*D] QKV row
    g = np.random.default_rng(4)
    T, H, D = 5, 2, 16
    qkv = g.standard_normal((T, 3 * H * D))
    q = qkv[:, :H * D].reshape(T, H, D)
    assert not q.flags.c_contiguous
    w = g.uniform(0.5, 1.5, D)
    pos = np.arange(T, dtype=np.int32)
    y = oracle.qk_norm_rope(q, w, pos, 1e-6, 10000.0, IL)
    y2 = oracle.qk_norm_rope(np.ascontiguousarray(q), w, pos, 1e-6, 10000.0, IL)
    np.testing.assert_array_equal(y, y2)


def test_sampled_rows_equal_full_run():
    w = wl.config(1)
    x = wl.prologue_inputs(w)
    y = oracle.qk_norm_rope(x["q"], x["w_q"], x["pos"], w.eps, w.rope_base, IL)
    rows = np.array([0, 7, 199, 200, 511], np.int32)
    ys = oracle.qk_norm_rope(x["q"], x["w_q"], x["pos"], w.eps, w.rope_base, IL, rows=rows)
    np.testing.assert_array_equal(ys, y[rows])
