"""Pins for the oracle's three-axis (t, h, w) RoPE variant (CPU only).

Reading (the pages give no RoPE variant): pair j keeps theta_j = base^(-2j/D)
and takes its position from the t, h or w id according to consecutive
sections of the D/2 pair indices. Pinned by reduction to the one-axis
oracle, a closed form, and the relative-position property per axis.
"""

import math

import numpy as np
import pytest

from oracle import oracle

IL, HALF = oracle.ROPE_INTERLEAVED, oracle.ROPE_HALF


def _x(seed, T, H, D):
    return np.random.default_rng(seed).standard_normal((T, H, D))


@pytest.mark.parametrize("style", [IL, HALF])
@pytest.mark.parametrize("sections", [(16, 24, 24), (32, 0, 32), (1, 62, 1)])
def test_equal_ids_reduce_to_one_axis_rope(style, sections):
    T, H, D = 7, 2, 128
    x = _x(1, T, H, D)
    w = np.random.default_rng(2).uniform(0.5, 1.5, D)
    pos = np.random.default_rng(3).integers(0, 60000, T).astype(np.int32)
    y3 = oracle.qk_norm_rope_3axis(x, w, np.stack([pos, pos, pos], 1), sections, 1e-6, 10000.0, style)
    y1 = oracle.qk_norm_rope(x, w, pos, 1e-6, 10000.0, style)
    np.testing.assert_allclose(y3, y1, atol=1e-13)


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_single_section_uses_that_axis_only(axis):
    T, H, D = 5, 1, 64
    x = _x(4, T, H, D)
    w = np.ones(D)
    pos3 = np.random.default_rng(5).integers(0, 5000, (T, 3)).astype(np.int32)
    sec = [0, 0, 0]
    sec[axis] = D // 2
    y3 = oracle.qk_norm_rope_3axis(x, w, pos3, sec, 1e-6, 10000.0, IL)
    y1 = oracle.qk_norm_rope(x, w, pos3[:, axis].copy(), 1e-6, 10000.0, IL)
    np.testing.assert_allclose(y3, y1, atol=1e-13)


def test_closed_form_two_pairs_two_tokens():
    # D = 4, sections (1, 1, 0): pair 0 (theta 1) turns by the t id, pair 1
    # (theta 10000^(-1/2) = 0.01) by the h id; the w id is unused.
    D = 4
    x = np.zeros((2, 1, D))
    x[:, 0, 0] = 1.0
    x[:, 0, 2] = 1.0
    pos3 = np.array([[3, 200, 7], [11, 50, 900]], np.int32)
    y = oracle.qk_norm_rope_3axis(x, np.ones(D), pos3, (1, 1, 0), 0.0, 10000.0, IL)
    r = math.sqrt(2.0)
    for i, (t, h, _) in enumerate(pos3):
        np.testing.assert_allclose(y[i, 0], [r * math.cos(t), r * math.sin(t),
                                             r * math.cos(0.01 * h), r * math.sin(0.01 * h)], atol=1e-12)


@pytest.mark.parametrize("style", [IL, HALF])
def test_dot_products_depend_on_the_position_difference_per_axis(style):
    H, D = 1, 64
    q, k = _x(6, 1, H, D), _x(7, 1, H, D)
    w = np.ones(D)
    sec = (8, 12, 12)
    for m, n in [((5, 40, 7), (2, 3, 1)), ((11, 47, 95), (3, 0, 90))]:
        m3, n3 = np.array([m], np.int32), np.array([n], np.int32)
        d3 = np.array([np.subtract(m, n)], np.int32)
        z3 = np.zeros((1, 3), np.int32)
        qm = oracle.qk_norm_rope_3axis(q, w, m3, sec, 1e-6, 10000.0, style)
        kn = oracle.qk_norm_rope_3axis(k, w, n3, sec, 1e-6, 10000.0, style)
        qd = oracle.qk_norm_rope_3axis(q, w, d3, sec, 1e-6, 10000.0, style)
        k0 = oracle.qk_norm_rope_3axis(k, w, z3, sec, 1e-6, 10000.0, style)
        assert abs(np.sum(qm * kn) - np.sum(qd * k0)) <= 1e-10


def test_rejects_sections_that_do_not_cover_the_pairs():
    x = np.zeros((1, 1, 8))
    with pytest.raises(ValueError):
        oracle.qk_norm_rope_3axis(x, np.ones(8), np.zeros((1, 3), np.int32), (1, 1, 1), 1e-6, 1e4)
    with pytest.raises(ValueError):
        oracle.qk_norm_rope_3axis(x, np.ones(8), np.zeros((1, 3), np.int32), (5, -1, 0), 1e-6, 1e4)
