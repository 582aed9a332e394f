"""Pins for the oracle's full-width Q/K norm + RoPE (CPU only): the RMS over
all H*D elements of a token (one weight per element) instead of per head.
A reading the pages leave open ("Q/K normalisation merged with RoPE",
"FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长", section "融合 DiT 算子")."""

import math

import numpy as np
import pytest

from oracle import oracle

IL, HALF = oracle.ROPE_INTERLEAVED, oracle.ROPE_HALF


def test_single_head_equals_per_head_norm():
    g = np.random.default_rng(0)
    x = g.standard_normal((9, 1, 64))
    w = g.uniform(0.5, 1.5, 64)
    pos = g.integers(0, 50000, 9).astype(np.int32)
    np.testing.assert_allclose(oracle.qk_fullc_norm_rope(x, w, pos, 1e-6, 1e4),
                               oracle.qk_norm_rope(x, w, pos, 1e-6, 1e4), atol=1e-13)


@pytest.mark.parametrize("style", [IL, HALF])
def test_heads_with_equal_rms_equal_per_head_norm(style):
    # every head a sign-flipped copy of one vector: each head's mean square
    # equals the token's, so both norms agree; weights tiled per head
    g = np.random.default_rng(1)
    T, H, D = 5, 3, 32
    base = g.standard_normal((T, 1, D))
    x = np.concatenate([base, -base, base], axis=1)
    wd = g.uniform(0.5, 1.5, D)
    pos = g.integers(0, 1000, T).astype(np.int32)
    np.testing.assert_allclose(oracle.qk_fullc_norm_rope(x, np.tile(wd, H), pos, 1e-6, 1e4, style),
                               oracle.qk_norm_rope(x, wd, pos, 1e-6, 1e4, style), atol=1e-13)


def test_unit_rms_over_the_whole_token_and_weight_per_element():
    g = np.random.default_rng(2)
    T, H, D, eps = 4, 5, 16, 0.02
    x = g.standard_normal((T, H, D)) * np.array([0.1, 1.0, 3.0, 0.5, 2.0])[None, :, None]
    w = g.uniform(0.5, 1.5, H * D)
    y = oracle.qk_fullc_norm_rope(x, w, np.zeros(T, np.int32), eps, 1e4)
    ms = (x.reshape(T, -1) ** 2).mean(-1)
    got = ((y.reshape(T, -1) / w) ** 2).mean(-1)
    np.testing.assert_allclose(got, ms / (ms + eps), rtol=1e-13)
    # heads keep their relative scale (a per-head norm would equalise them)
    rms_h = np.sqrt((y / w.reshape(H, D)) ** 2).mean(-1)
    assert rms_h[0, 4] > 3 * rms_h[0, 0]


def test_constant_token_closed_form():
    H, D = 2, 4
    x = np.full((1, H, D), 2.0)
    w = np.arange(1, H * D + 1, dtype=np.float64)
    y = oracle.qk_fullc_norm_rope(x, w, np.zeros(1, np.int32), 5.0, 1e4)
    np.testing.assert_allclose(y.reshape(-1), w * 2.0 / 3.0, rtol=1e-15)   # 2 / sqrt(4 + 5)
