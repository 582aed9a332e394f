"""Pins for the oracle's fused adaLN modulation + gated residual + SwiGLU
(CPU only).

The pages list modulation, normalisation, residual connections and SwiGLU
among the fused DiT operators, with SwiGLU replacing a separate SiLU and
multiply ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长", section
"融合 DiT 算子"; "MiniMax H3 FastH3 real-time serving with vLLM-Omni", bullet
"Fused DiT operators"). Pinned by closed forms of SiLU, RMS/Layer norm and
the modulation, and by per-request lookup of the modulation vectors.
"""

import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import workloads as wl


def _zeros(B, C):
    return np.zeros((B, C), np.float32)


def _cu(T):
    return np.array([0, T], np.int32)


def test_silu_closed_forms():
    gate = np.array([[0.0, 1.0, 30.0, -30.0, 2.0]])
    up = np.array([[1.0, 1.0, 1.0, 1.0, 0.5]])
    x = np.ones((1, 4))
    _, _, act = oracle.modulate_swiglu(x, _zeros(1, 4), _zeros(1, 4), _zeros(1, 4), _cu(1),
                                       gate=gate, up=up)
    assert act[0, 0] == 0.0
    assert abs(act[0, 1] - 0.7310585786300049) <= 1e-16      # 1 / (1 + e^-1)
    assert abs(act[0, 2] - 30.0) <= 30.0 * 1e-12             # silu(x) -> x
    assert abs(act[0, 3]) <= 30.0 * math.exp(-30.0) * 1.01   # silu(x) -> 0
    assert abs(act[0, 4] - 0.5 * 2.0 / (1.0 + math.exp(-2.0))) <= 1e-15


def test_gate_is_the_silu_operand_and_up_the_multiplier():
    # silu(1) * 2 = 1.4621...; swapping operands would give silu(2) * 1 = 1.7616...
    _, _, act = oracle.modulate_swiglu(np.ones((1, 2)), _zeros(1, 2), _zeros(1, 2), _zeros(1, 2), _cu(1),
                                       gate=np.array([[1.0]]), up=np.array([[2.0]]))
    assert abs(act[0, 0] - 2.0 / (1.0 + math.exp(-1.0))) <= 1e-15


def test_rms_norm_of_constant_row_and_zero_modulation():
    C = 16
    x = np.full((1, C), 3.0)
    _, h, _ = oracle.modulate_swiglu(x, _zeros(1, C), _zeros(1, C), _zeros(1, C), _cu(1), eps=7.0)
    np.testing.assert_allclose(h, 3.0 / 4.0, rtol=1e-15)     # 3 / sqrt(9 + 7)


def test_layer_norm_closed_form():
    x = np.array([[1.0, 2.0, 3.0, 6.0]])                     # mean 3, biased var 3.5
    _, h, _ = oracle.modulate_swiglu(x, _zeros(1, 4), _zeros(1, 4), _zeros(1, 4), _cu(1),
                                     norm_type=oracle.NORM_LAYER, eps=0.5)
    np.testing.assert_allclose(h[0], (x[0] - 3.0) / 2.0, rtol=1e-15)


def test_none_norm_with_zero_modulation_is_identity_and_modulation_closed_form():
    g = np.random.default_rng(0)
    T, C = 5, 8
    x = g.standard_normal((T, C))
    _, h, _ = oracle.modulate_swiglu(x, _zeros(1, C), _zeros(1, C), _zeros(1, C), _cu(T),
                                     norm_type=oracle.NORM_NONE)
    np.testing.assert_array_equal(h, x)
    shift = g.standard_normal((1, C)).astype(np.float32)
    scale = g.standard_normal((1, C)).astype(np.float32)
    _, h, _ = oracle.modulate_swiglu(x, shift, scale, _zeros(1, C), _cu(T), norm_type=oracle.NORM_NONE)
    np.testing.assert_allclose(h, x * (1.0 + scale.astype(np.float64)) + shift.astype(np.float64), rtol=1e-15)


def test_rms_unit_before_modulation():
    g = np.random.default_rng(1)
    T, C, eps = 7, 64, 1e-3
    x = g.standard_normal((T, C)) * 0.1
    _, h, _ = oracle.modulate_swiglu(x, _zeros(1, C), _zeros(1, C), _zeros(1, C), _cu(T), eps=eps)
    ms = (x ** 2).mean(-1)
    np.testing.assert_allclose((h ** 2).mean(-1), ms / (ms + eps), rtol=1e-13)


def test_gated_residual_is_x_plus_gate_times_branch():
    g = np.random.default_rng(2)
    T, C = 4, 8
    x = g.standard_normal((T, C))
    br = g.standard_normal((T, C))
    gr = g.standard_normal((1, C)).astype(np.float32)
    xo, h, _ = oracle.modulate_swiglu(x, _zeros(1, C), _zeros(1, C), gr, _cu(T), branch=br,
                                      norm_type=oracle.NORM_NONE)
    np.testing.assert_allclose(xo, x + gr.astype(np.float64) * br, rtol=1e-15)
    np.testing.assert_array_equal(h, xo)                      # NONE, zero modulation


def test_modulation_vectors_follow_each_token_request():
    T, C = 10, 4
    x = np.ones((T, C))
    cu = np.array([0, 3, 3, 10], np.int32)                    # empty middle request
    shift = np.array([[1, 1, 1, 1], [50, 50, 50, 50], [2, 2, 2, 2]], np.float32)
    _, h, _ = oracle.modulate_swiglu(x, shift, _zeros(3, C), _zeros(3, C), cu, norm_type=oracle.NORM_NONE)
    np.testing.assert_array_equal(h[:3], 2.0)
    np.testing.assert_array_equal(h[3:], 3.0)


def test_sampled_rows_equal_full_run_on_tiny_config():
    w = wl.config(1)
    e = wl.epilogue_inputs(w, with_branch=True)
    full = oracle.modulate_swiglu(e["x"], e["shift"], e["scale"], e["gate_res"], e["cu_seqlens"],
                                  branch=e["branch"], gate=e["gate"], up=e["up"])
    rows = np.array([0, 199, 200, 511], np.int32)
    part = oracle.modulate_swiglu(e["x"], e["shift"], e["scale"], e["gate_res"], e["cu_seqlens"],
                                  branch=e["branch"], gate=e["gate"], up=e["up"], rows=rows)
    for a, b in zip(full, part):
        np.testing.assert_array_equal(a[rows], b)
