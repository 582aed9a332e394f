"""Pins for the oracle's packed varlen attention (CPU only).

The oracle is checked against things other than itself: an independently
written dense padded-and-masked brute force, closed forms, and invariants of
softmax attention over one packed sequence per request ("FastH3 在八卡 B300
上实现完整 MP4 生成快于播放时长", section "长序列注意力与通信优化": requests are
packed into one long sequence and only valid tokens are processed).
"""

import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import workloads as wl
from tests.bruteforce import padded_masked_attention


def _rand(seed, T, H, D):
    g = np.random.default_rng(seed)
    return [g.standard_normal((T, H, D)) for _ in range(3)]


@pytest.mark.parametrize("lens", [[1], [2], [3], [17], [128], [129], [300], [5, 0, 17, 1], [0, 64, 0]])
def test_matches_bruteforce_f64(lens):
    H, D = 2, 16
    T = sum(lens)
    q, k, v = _rand(sum(lens) + len(lens), T, H, D)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.varlen_attn(q, k, v, cu, scale)
    ob, lb = padded_masked_attention(q, k, v, cu, scale)
    assert np.max(np.abs(o - ob)) <= 1e-12
    assert np.max(np.abs(lse - lb)) <= 1e-12


def test_matches_bruteforce_on_tiny_config_bf16():
    w = wl.config(1)
    x = wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(w.D)
    o, lse = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], scale)
    f = wl.bf16_bits_to_f64
    ob, lb = padded_masked_attention(f(x["q"]), f(x["k"]), f(x["v"]), x["cu_seqlens"], scale)
    assert np.max(np.abs(o - ob)) <= 1e-12
    assert np.max(np.abs(lse - lb)) <= 1e-12


def test_zero_query_gives_segment_mean_and_log_length():
    lens = [7, 30]
    T, H, D = sum(lens), 3, 8
    _, k, v = _rand(1, T, H, D)
    q = np.zeros((T, H, D))
    cu = np.array([0, 7, 37], np.int32)
    o, lse = oracle.varlen_attn(q, k, v, cu, 0.37)
    for b in range(2):
        seg = slice(cu[b], cu[b + 1])
        np.testing.assert_allclose(o[seg], np.broadcast_to(v[seg].mean(axis=0), o[seg].shape), atol=1e-14)
        np.testing.assert_allclose(lse[seg], math.log(lens[b]), atol=1e-14)


def test_equal_keys_give_mean_of_values():
    T, H, D = 11, 2, 4
    q, _, v = _rand(2, T, H, D)
    k = np.ones((T, H, D)) * 0.5
    o, _ = oracle.varlen_attn(q, k, v, np.array([0, T], np.int32), 1.0)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-13)


def test_length_one_segment_returns_its_value_and_score():
    T, H, D = 4, 2, 8
    q, k, v = _rand(3, T, H, D)
    cu = np.array([0, 1, 2, 3, 4], np.int32)
    scale = 0.25
    o, lse = oracle.varlen_attn(q, k, v, cu, scale)
    np.testing.assert_allclose(o, v, atol=1e-15)
    np.testing.assert_allclose(lse, scale * np.einsum("thd,thd->th", q, k), atol=1e-13)


def test_two_key_closed_form_pins_scale_and_operand_order():
    # q = e0, k0 = a*e0, k1 = 0: scores (a*scale, 0); softmax weights
    # w0 = e^{a s} / (e^{a s} + 1); o = w0 v0 + (1 - w0) v1.
    D, a, scale = 4, 3.0, 0.5
    q = np.zeros((2, 1, D)); q[:, 0, 0] = 1.0
    k = np.zeros((2, 1, D)); k[0, 0, 0] = a
    v = np.zeros((2, 1, D)); v[0, 0] = [1, 2, 3, 4]; v[1, 0] = [-1, 0, 5, 2]
    o, lse = oracle.varlen_attn(q, k, v, np.array([0, 2], np.int32), scale)
    w0 = math.exp(a * scale) / (math.exp(a * scale) + 1.0)
    expect = w0 * v[0, 0] + (1 - w0) * v[1, 0]
    np.testing.assert_allclose(o[0, 0], expect, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], math.log(math.exp(a * scale) + 1.0), atol=1e-15)


def test_one_dominant_key_selects_its_value_row():
    T, H, D = 50, 2, 16
    g = np.random.default_rng(4)
    q = g.standard_normal((T, H, D)) * 0.01
    k = g.standard_normal((T, H, D)) * 0.01
    v = g.standard_normal((T, H, D))
    hot = 31
    q[:, :, 0] = 1.0
    k[hot, :, 0] = 200.0
    o, _ = oracle.varlen_attn(q, k, v, np.array([0, T], np.int32), 1.0)
    np.testing.assert_allclose(o, np.broadcast_to(v[hot], o.shape), atol=1e-12)


def test_joint_permutation_of_keys_and_values_inside_a_segment():
    lens = [40, 25]
    T, H, D = 65, 2, 8
    q, k, v = _rand(5, T, H, D)
    cu = np.array([0, 40, 65], np.int32)
    perm = np.arange(T)
    g = np.random.default_rng(6)
    perm[:40] = g.permutation(40)
    perm[40:] = 40 + g.permutation(25)
    o1, l1 = oracle.varlen_attn(q, k, v, cu, 0.3)
    o2, l2 = oracle.varlen_attn(q, k[perm], v[perm], cu, 0.3)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_packed_equals_segments_run_one_by_one():
    lens = [13, 1, 0, 29, 8]
    T, H, D = sum(lens), 3, 8
    q, k, v = _rand(7, T, H, D)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, lse = oracle.varlen_attn(q, k, v, cu, 0.2)
    for b, L in enumerate(lens):
        if L == 0:
            continue
        s = slice(cu[b], cu[b + 1])
        ob, lb = oracle.varlen_attn(q[s], k[s], v[s], np.array([0, L], np.int32), 0.2)
        np.testing.assert_allclose(o[s], ob, atol=1e-14)
        np.testing.assert_allclose(lse[s], lb, atol=1e-14)


def test_packed_equals_padded_and_masked():
    # each request padded to the batch maximum with junk rows that the key
    # mask must exclude: large keys and huge values would dominate if leaked
    lens = [30, 50, 7]
    H, D = 2, 8
    T = sum(lens)
    q, k, v = _rand(8, T, H, D)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, lse = oracle.varlen_attn(q, k, v, cu, 0.4)
    Lmax = max(lens)
    Qp = np.full((3, Lmax, H, D), 3.0)
    Kp = np.full((3, Lmax, H, D), 50.0)
    Vp = np.full((3, Lmax, H, D), 1e6)
    for b, L in enumerate(lens):
        Qp[b, :L], Kp[b, :L], Vp[b, :L] = q[cu[b]:cu[b + 1]], k[cu[b]:cu[b + 1]], v[cu[b]:cu[b + 1]]
    from tests.bruteforce import attention_padded
    Op, Lp = attention_padded(Qp, Kp, Vp, lens, 0.4)
    for b, L in enumerate(lens):
        np.testing.assert_allclose(o[cu[b]:cu[b + 1]], Op[b, :L], atol=1e-12)
        np.testing.assert_allclose(lse[cu[b]:cu[b + 1]], Lp[b, :, :L].T, atol=1e-12)


def test_sampled_rows_equal_full_run():
    w = wl.config(1)
    x = wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(w.D)
    o, lse = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], scale)
    rows = wl.sample_rows(w, per_segment=16)
    os_, ls = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, rows=rows)
    np.testing.assert_array_equal(os_, o[rows])
    np.testing.assert_array_equal(ls, lse[rows])


def test_rejects_bad_cu_seqlens():
    q = np.zeros((4, 1, 2))
    with pytest.raises(ValueError):
        oracle.varlen_attn(q, q, q, np.array([0, 3, 2, 4], np.int32), 1.0)
    with pytest.raises(ValueError):
        oracle.varlen_attn(q, q, q, np.array([0, 3], np.int32), 1.0)
