"""Pins for the oracle's FP8 (e4m3) quantisation and the attention with Q and
K in FP8 (CPU only).

SAGE quantises the attention computation to FP8 ("FastH3 在八卡 B300 上实现
完整 MP4 生成快于播放时长", bullet on TRTLLM_ATTN SAGE and Skip-Softmax). The
quantisation here is a reading: per-head absmax scaling of Q and K to the
e4m3 range (amax -> 448), nearest-even rounding. Checked against torch's
float8_e4m3fn conversion (a library routine), the format's own code table,
error bounds of a 3-bit mantissa, exact cases, and a dense brute force on
the dequantised inputs.
"""

import math

import numpy as np
import pytest
import torch

from oracle import oracle
from tests.bruteforce import padded_masked_attention


def e4m3_table():
    """The 254 finite e4m3 values, from torch's decoder (codes 0x00..0xFF
    without the two NaN codes)."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    return codes, vals


def test_codes_match_torch_conversion():
    g = np.random.default_rng(0)
    x = np.concatenate([g.uniform(-448, 448, 100000), g.standard_normal(100000) * 0.01, g.standard_normal(50000) * 5,
                        [0.0, -0.0, 448.0, -448.0, 460.0, 1e-3, 2.0 ** -10, 3 * 2.0 ** -10, 1.5 * 2.0 ** -9,
                         2.5 * 2.0 ** -9, 1.0625, 1.1875, 1.0625 * 2.0 ** -6, 7.5 * 2.0 ** -9]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_codes(x), ref)


def test_every_code_round_trips_and_midpoints_go_to_even():
    codes, vals = e4m3_table()
    assert np.array_equal(oracle.e4m3_codes(vals), codes)
    # midpoints between neighbouring positive values round to the even code
    pos = np.sort(vals[vals > 0])
    mid = ((pos[:-1].astype(np.float64) + pos[1:]) / 2).astype(np.float32)
    got = oracle.e4m3_codes(mid)
    lo = oracle.e4m3_codes(pos[:-1])
    hi = oracle.e4m3_codes(pos[1:])
    assert np.array_equal(got, np.where(lo % 2 == 0, lo, hi))


def test_saturation_beyond_448():
    x = np.array([464.0, 500.0, 1e6, -600.0, 3.0e38], np.float32)
    assert list(oracle.e4m3_codes(x)) == [0x7E, 0x7E, 0x7E, 0xFE, 0x7E]


def _decode(c):
    return torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def test_per_head_quantisation_bounds_and_independence():
    g = np.random.default_rng(1)
    T, H, D = 300, 3, 16
    x = g.standard_normal((T, H, D))
    x[:, 1] *= 1000.0
    x[:, 2] = 0.0
    codes, deq = oracle.quantize_e4m3(x)
    amax = np.abs(x).max(axis=(0, 2))
    assert deq[0] == np.float32(np.float32(amax[0]) / np.float32(448.0)) and deq[2] == 1.0
    assert np.all(codes[:, 2] == 0)
    back = _decode(codes) * deq[None, :, None]
    # 3 stored mantissa bits: relative error <= 2^-4 in the normal range,
    # absolute error <= 2^-10 * deq below it
    err = np.abs(back - x)
    assert np.all(err <= np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * deq[None, :, None]) * (1 + 1e-6))
    # the element with the largest magnitude maps to +-448
    t, d = np.unravel_index(np.argmax(np.abs(x[:, 0])), (T, D))
    assert codes[t, 0, d] in (0x7E, 0xFE)
    # head 0's codes do not depend on head 1's scale
    x2 = x.copy()
    x2[:, 1] *= 0.001
    assert np.array_equal(oracle.quantize_e4m3(x2)[0][:, 0], codes[:, 0])


def test_exact_when_inputs_are_e4m3_values_with_absmax_448():
    codes, vals = e4m3_table()
    g = np.random.default_rng(2)
    T, H, D = 200, 2, 16
    q = g.choice(vals, (T, H, D)).astype(np.float64) * 0.25
    k = g.choice(vals, (T, H, D)).astype(np.float64) * 0.5
    q[0, :, 0] = 448.0 * 0.25
    k[0, :, 0] = 448.0 * 0.5
    v = g.standard_normal((T, H, D))
    cu = np.array([0, 77, 200], np.int32)
    o, lse, q8, k8, deq = oracle.varlen_attn_fp8qk(q, k, v, cu, 0.1)
    assert np.allclose(deq, [0.25, 0.25, 0.5, 0.5], rtol=0, atol=0)
    ob, lb = oracle.varlen_attn(q, k, v, cu, 0.1)
    assert np.max(np.abs(o - ob)) <= 1e-12 and np.max(np.abs(lse - lb)) <= 1e-12


def test_matches_bruteforce_on_dequantised_inputs():
    g = np.random.default_rng(3)
    T, H, D = 257, 2, 32
    q, k, v = (g.standard_normal((T, H, D)) for _ in range(3))
    cu = np.array([0, 1, 130, 257], np.int32)
    scale = 1.0 / math.sqrt(D)
    o, lse, q8, k8, deq = oracle.varlen_attn_fp8qk(q, k, v, cu, scale)
    qd = _decode(q8) * deq[None, :H, None]
    kd = _decode(k8) * deq[None, H:, None]
    ob, lb = padded_masked_attention(qd, kd, v, cu, scale)
    assert np.max(np.abs(o - ob)) <= 1e-12 and np.max(np.abs(lse - lb)) <= 1e-12
    # and it is not the unquantised attention
    op, _ = oracle.varlen_attn(q, k, v, cu, scale)
    assert np.max(np.abs(o - op)) > 1e-4


def test_sampled_rows_equal_full_evaluation():
    g = np.random.default_rng(4)
    T, H, D = 300, 2, 16
    q, k, v = (g.standard_normal((T, H, D)) for _ in range(3))
    cu = np.array([0, 300], np.int32)
    o, lse, q8, _, _ = oracle.varlen_attn_fp8qk(q, k, v, cu, 0.25)
    rows = np.array([0, 5, 299], np.int32)
    o2, l2, q82, _, _ = oracle.varlen_attn_fp8qk(q, k, v, cu, 0.25, rows=rows)
    assert np.array_equal(o2, o[rows]) and np.array_equal(l2, lse[rows]) and np.array_equal(q82, q8)


def test_fp8_with_block_skipping_is_skipping_on_the_dequantised_inputs():
    # composition: FP8 Q K^T with a finite tau = the block-skipping oracle on
    # the dequantised Q, K (decoded by torch); tau = inf = no skipping
    g = np.random.default_rng(6)
    T, H, D = 900, 2, 32
    q = g.standard_normal((T, H, D)) * 2.5
    k = g.standard_normal((T, H, D)) * np.repeat(g.choice([0.02, 3.0], math.ceil(T / 128)), 128)[:T, None, None]
    v = g.standard_normal((T, H, D))
    cu = np.array([0, 400, T], np.int32)
    scale = 1.0 / math.sqrt(D)
    counts = []
    o, lse, q8, k8, deq = oracle.varlen_attn_fp8qk(q, k, v, cu, scale, tau=6.0, skip_block=(16, 64),
                                                   skip_tile_rows=64, counts_out=counts)
    qd = _decode(q8) * deq[None, :H, None]
    kd = _decode(k8) * deq[None, H:, None]
    os_, ls, cs = oracle.varlen_attn_skip(qd, kd, v, cu, scale, 6.0, block=(16, 64), tile_rows=64)
    assert counts == [cs] and cs[0] > 0
    assert np.array_equal(o, os_) and np.array_equal(lse, ls)
    o_inf, _, _, _, _ = oracle.varlen_attn_fp8qk(q, k, v, cu, scale)
    on, _, _, _, _ = oracle.varlen_attn_fp8qk(q, k, v, cu, scale, tau=math.inf)
    assert np.array_equal(o_inf, on)
    with pytest.raises(ValueError):
        oracle.varlen_attn_fp8qk(q, k, v, cu, scale, tau=6.0)  # a finite tau needs the block geometry


# ---------------------------------------------------------------- Q, K, V and P in FP8
#
# The definition: p_j = exp(s_j - m) against the row's exact maximum m,
# e4m3(p_j) in the numerator, p_j in the denominator. The online schedule
# (oracle.varlen_attn_fp8_online) rounds each p against the running maximum
# of a streaming implementation instead; it is pinned separately below, and
# against the definition by the bound that follows from e4m3's step.


def _one_row_case(k_vals, v_vals, scale, online=None):
    """One request, one head, D = 1, q = 1.75: keys k_vals, values v_vals.
    Every tensor's amax is 1.75 = 448 * 2^-8, so its scale is exactly 2^-8
    and values that are e4m3 codes times 2^-8 quantise exactly."""
    L = len(k_vals)
    q = np.full((L, 1, 1), 1.75)
    k = np.array(k_vals, np.float64).reshape(L, 1, 1)
    v = np.array(v_vals, np.float64).reshape(L, 1, 1)
    cu = np.array([0, L], np.int32)
    if online is None:
        o, lse, _ = oracle.varlen_attn_fp8(q, k, v, cu, scale)
    else:
        o, lse, _ = oracle.varlen_attn_fp8_online(q, k, v, cu, scale, kblock=online[0], threshold=online[1])
    return o[0, 0, 0], lse[0, 0]


def test_fp8_p_rounds_in_the_numerator_only():
    # keys 1.75 and 0.875 at scale 0.6 ln 2 / 1.75^2: u = (0.6, 0.3),
    # p = (1, 2^-0.3) and e4m3(2^-0.3 = 0.81225) = 0.8125 (13/16); values
    # 1.75 and -1.75
    o, lse = _one_row_case([1.75, 0.875], [1.75, -1.75], 0.6 * math.log(2.0) / 1.75 ** 2)
    p2 = 2.0 ** -0.3
    assert abs(o - 1.75 * (1.0 - 0.8125) / (1.0 + p2)) <= 1e-12
    assert abs(lse - (0.6 + math.log2(1.0 + p2)) * math.log(2.0)) <= 1e-12


def test_fp8_p_is_rounded_against_the_rows_exact_maximum():
    # keys 0 and 1.75 at scale 5.3 ln 2 / 1.75^2: u = (0, 5.3); the maximum is
    # the second key, so p = (2^-5.3, 1) and e4m3(2^-5.3 = 0.025383) =
    # 1.625 * 2^-6 = 0.025390625. Rounding against the first key instead would
    # give p = (1, 2^5.3 -> 40): a different numerator.
    o, lse = _one_row_case([0.0, 1.75], [1.75, -1.75], 5.3 * math.log(2.0) / 1.75 ** 2)
    p1 = 2.0 ** -5.3
    assert abs(o - 1.75 * (0.025390625 - 1.0) / (p1 + 1.0)) <= 1e-12
    assert abs(lse - (5.3 + math.log2(1.0 + p1)) * math.log(2.0)) <= 1e-12


def test_fp8_small_probabilities_round_on_the_subnormal_grid():
    # keys 1.75, 0.75, 0 at scale 7.5 ln 2 / 1.75: u = (13.125, 5.625, 0), so
    # p = (1, 2^-7.5, 2^-13.125). Below 2^-6 e4m3 steps by 2^-9: 2^-7.5 =
    # 2.83 * 2^-9 rounds to 3 * 2^-9 and 2^-13.125 (0.11 steps) to 0, while the
    # denominator keeps all three; values 0.5, 1.75, -1.75
    o, lse = _one_row_case([1.75, 0.75, 0.0], [0.5, 1.75, -1.75], 7.5 * math.log(2.0) / 1.75)
    den = 1.0 + 2.0 ** -7.5 + 2.0 ** -13.125
    assert abs(o - (0.5 + 3 * 2.0 ** -9 * 1.75) / den) <= 1e-12
    assert abs(lse - (13.125 + math.log2(den)) * math.log(2.0)) <= 1e-12


def test_fp8_is_exact_on_representable_inputs():
    # Q, K entries in {0, 1} on dims 2.. with one 1.75 on dims 0 / 1 where the
    # other tensor is 0 (amax 1.75 -> scale 2^-8 exactly), scale ln 2: integer
    # log2 scores in [0, 6], so every p is a power of two e4m3 holds; V from
    # e4m3 values times 2^-6 with amax 7 (scale 2^-6): the FP8 attention then
    # equals the plain attention
    g = np.random.default_rng(8)
    T, H, D = 400, 2, 8
    q = np.zeros((T, H, D))
    k = np.zeros((T, H, D))
    q[:, :, 2:] = g.integers(0, 2, (T, H, D - 2))
    k[:, :, 2:] = g.integers(0, 2, (T, H, D - 2))
    q[0, :, 0] = 1.75
    k[0, :, 1] = 1.75
    _, vals = e4m3_table()
    v = g.choice(vals[np.abs(vals) <= 448], (T, H, D)).astype(np.float64) * 2.0 ** -6
    v[0, :, 0] = 7.0
    cu = np.array([0, 150, 400], np.int32)
    o, lse, deq = oracle.varlen_attn_fp8(q, k, v, cu, math.log(2.0))
    assert np.array_equal(deq, np.array([2.0 ** -8] * 4 + [2.0 ** -6] * 2, np.float32))
    ob, lb = oracle.varlen_attn(q, k, v, cu, math.log(2.0))
    assert np.max(np.abs(o - ob)) <= 1e-12 and np.max(np.abs(lse - lb)) <= 1e-12


def _dequantised(q, k, v):
    return [_decode(c) * d[None, :, None] for c, d in (oracle.quantize_e4m3(x) for x in (q, k, v))]


def _row_weights(qd, kd, cu, scale, t, h):
    """Exact-max probabilities p_j of row t, head h over its request."""
    i = int(np.searchsorted(cu, t, side="right") - 1)
    s = scale * (kd[cu[i]:cu[i + 1], h] @ qd[t, h])
    return np.exp(s - s.max()), int(cu[i]), int(cu[i + 1])


def test_fp8_error_bound_against_exact_p():
    # e4m3 rounds p <= 1 to within 2^-4 p in its normal range and within 2^-10
    # below it, so every element of O lies within
    # sum_j max(2^-4 p_j, 2^-10) |v_j| / sum_j p_j of the attention with exact P
    # on the same dequantised Q, K, V
    g = np.random.default_rng(9)
    T, H, D = 500, 2, 32
    q, k, v = (g.standard_normal((T, H, D)) for _ in range(3))
    cu = np.array([0, 130, 500], np.int32)
    scale = 1.0 / math.sqrt(D)
    o, _, _ = oracle.varlen_attn_fp8(q, k, v, cu, scale)
    qd, kd, vd = _dequantised(q, k, v)
    ob, _ = padded_masked_attention(qd, kd, vd, cu, scale)
    assert np.max(np.abs(o - ob)) > 0
    for t in range(0, T, 7):
        for h in range(H):
            p, lo, hi = _row_weights(qd, kd, cu, scale, t, h)
            bound = (np.maximum(2.0 ** -4 * p, 2.0 ** -10)[:, None] * np.abs(vd[lo:hi, h])).sum(0) / p.sum()
            assert np.all(np.abs(o[t, h] - ob[t, h]) <= bound * (1 + 1e-9) + 1e-15)


def test_fp8_sampled_rows_equal_full_evaluation():
    g = np.random.default_rng(10)
    T, H, D = 300, 2, 16
    q, k, v = (g.standard_normal((T, H, D)) for _ in range(3))
    cu = np.array([0, 17, 300], np.int32)
    o, lse, _ = oracle.varlen_attn_fp8(q, k, v, cu, 0.25)
    rows = np.array([0, 16, 17, 150, 299], np.int32)
    o2, l2, _ = oracle.varlen_attn_fp8(q, k, v, cu, 0.25, rows=rows)
    assert np.array_equal(o2, o[rows]) and np.array_equal(l2, lse[rows])


# ----------------------------------------------- the online schedule of the same FP8 attention

@pytest.mark.parametrize("kblock, threshold", [(128, 8.0), (64, 4.0)])
def test_online_running_maximum_moves_only_beyond_the_threshold(kblock, threshold):
    # kblock keys with k = 0 (block 0, u = 0), then one key with k = 1.75
    # (block 1) whose u is threshold - 2.7: within the threshold, so m stays
    # 0 and p = 2^u is rounded as it is (2^5.3 = 39.40 -> 40, 2^1.3 = 2.462 ->
    # 2.5); values 0 then 1.75
    u = threshold - 2.7
    k = [0.0] * kblock + [1.75]
    o, _ = _one_row_case(k, [0.0] * kblock + [1.75], u * math.log(2.0) / 1.75 ** 2, online=(kblock, threshold))
    rounded = {8.0: 40.0, 4.0: 2.5}[threshold]
    assert abs(o - 1.75 * rounded / (kblock + 2.0 ** u)) <= 1e-12
    # u = threshold + 1.3 is beyond it: m moves, block 0's sums scale by 2^-u
    # and the new key has p = 1 exactly; block-0 values 0.5
    u = threshold + 1.3
    o, _ = _one_row_case(k, [0.5] * kblock + [1.75], u * math.log(2.0) / 1.75 ** 2, online=(kblock, threshold))
    a = 2.0 ** -u
    assert abs(o - (kblock * 0.5 * a + 1.75) / (kblock * a + 1.0)) <= 1e-12


def test_online_with_one_block_per_request_is_the_definition():
    g = np.random.default_rng(12)
    T, H, D = 400, 2, 32
    q, k, v = (g.standard_normal((T, H, D)) * 2 for _ in range(3))
    cu = np.array([0, 150, 400], np.int32)
    o, lse, d = oracle.varlen_attn_fp8(q, k, v, cu, 0.2)
    for threshold in (0.0, 8.0):
        o2, l2, d2 = oracle.varlen_attn_fp8_online(q, k, v, cu, 0.2, kblock=256, threshold=threshold)
        assert np.array_equal(d, d2)
        assert np.max(np.abs(o - o2)) <= 1e-12 and np.max(np.abs(lse - l2)) <= 1e-12


@pytest.mark.parametrize("kblock, threshold", [(128, 8.0), (32, 2.0)])
def test_online_schedule_against_the_definition_bound(kblock, threshold):
    # each p is rounded against a maximum that is never above the row's: both
    # roundings lie within max(2^-4 p, 2^-10) of p (in units of the row's
    # maximum), so they differ by at most max(2^-3 p, 2^-9); with P in the
    # numerator only, O differs by at most sum_j max(2^-3 p_j, 2^-9) |v_j| / l.
    # The lse is the same sum either way.
    g = np.random.default_rng(13)
    T, H, D = 600, 2, 32
    q, k, v = (g.standard_normal((T, H, D)) for _ in range(3))
    k[300:, :, :] *= 2.0  # later keys score higher: the running maximum lags
    cu = np.array([0, 90, 600], np.int32)
    scale = 1.0 / math.sqrt(D)
    o, lse, _ = oracle.varlen_attn_fp8(q, k, v, cu, scale)
    o2, l2, _ = oracle.varlen_attn_fp8_online(q, k, v, cu, scale, kblock=kblock, threshold=threshold)
    assert np.max(np.abs(o - o2)) > 0 and np.max(np.abs(lse - l2)) <= 1e-12
    qd, kd, vd = _dequantised(q, k, v)
    for t in range(0, T, 5):
        for h in range(H):
            p, lo, hi = _row_weights(qd, kd, cu, scale, t, h)
            bound = (np.maximum(2.0 ** -3 * p, 2.0 ** -9)[:, None] * np.abs(vd[lo:hi, h])).sum(0) / p.sum()
            assert np.all(np.abs(o[t, h] - o2[t, h]) <= bound * (1 + 1e-9) + 1e-15)


def test_online_schedule_arguments_are_validated():
    x = np.zeros((4, 1, 8))
    cu = np.array([0, 4], np.int32)
    for kb, th in [(0, 8.0), (128, -1.0), (128, float("nan"))]:
        with pytest.raises(ValueError):
            oracle.varlen_attn_fp8_online(x, x, x, cu, 1.0, kblock=kb, threshold=th)


# ----------------------------------------------- FP8 P with block skipping (Skip-Softmax)

def _skip_case(kb, qr, seed=0):
    """One request of four key blocks of kb keys, one head, D = 16: queries
    close to +a*u, keys of blocks 0 and 2 close to -a*u (block 2 is dropped,
    block 0 never is), except query row qr + 5, which points at -u, so its
    query block keeps block 2. Dimension 15 is zero everywhere but in token
    0, which holds every tensor's absolute maximum there: removing block 2's
    tokens leaves all three quantisation scales unchanged."""
    L, D, a = 4 * kb, 16, 6.0
    g = np.random.default_rng(seed)
    u = np.zeros(D)
    u[0] = 1.0
    q = a * u + 0.1 * g.standard_normal((L, D))
    k = 0.3 * g.standard_normal((L, D))
    k[2 * kb:3 * kb] -= a * u
    k[0:kb] -= a * u
    q[qr + 5] = -a * u + 0.1 * g.standard_normal(D)
    v = g.standard_normal((L, D))
    for x in (q, k, v):
        x[:, 15] = 0.0
        x[0, 15] = 20.0
    return q[:, None, :], k[:, None, :], v[:, None, :], np.array([0, L], np.int32), 1.0 / math.sqrt(D)


@pytest.mark.parametrize("geom", [(16, 64, 64), (32, 128, 128)])
def test_fp8_skipping_is_the_definition_over_the_kept_keys(geom):
    # rows whose query block drops key block 2 equal the FP8 attention of the
    # same sequence with block 2's tokens removed; rows of the query block
    # that keeps it equal the FP8 attention of the whole sequence; the counts
    # are the forced ones, and the same as the FP8 Q K^T composition's
    qr, kb, tile = geom
    q, k, v, cu, scale = _skip_case(kb, qr)
    L = q.shape[0]
    counts = []
    o, lse, _ = oracle.varlen_attn_fp8(q, k, v, cu, scale, tau=10.0, skip_block=(qr, kb), skip_tile_rows=tile,
                                       counts_out=counts)
    assert counts == [(L // qr - 1, math.ceil(L / tile) - 1)]
    qk_counts = []
    oracle.varlen_attn_fp8qk(q, k, v, cu, scale, tau=10.0, skip_block=(qr, kb), skip_tile_rows=tile,
                             counts_out=qk_counts)
    assert qk_counts == counts
    full, full_lse, _ = oracle.varlen_attn_fp8(q, k, v, cu, scale)
    keep = np.r_[0:2 * kb, 3 * kb:L]
    red, red_lse, _ = oracle.varlen_attn_fp8(q[keep], k[keep], v[keep], np.array([0, len(keep)], np.int32), scale)
    pos_in_red = {int(t): i for i, t in enumerate(keep)}
    for t in range(L):
        if qr <= t < 2 * qr:
            ref, ref_lse = full[t], full_lse[t]
        elif t in pos_in_red:
            ref, ref_lse = red[pos_in_red[t]], red_lse[pos_in_red[t]]
        else:
            continue  # a row of block 2 itself: its own request has no reduced counterpart
        np.testing.assert_allclose(o[t], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[t], ref_lse, rtol=0, atol=1e-12)
    # row qr + 5 attends mostly to block 2: dropping it would change its output
    assert np.max(np.abs(full[qr + 5] - red[pos_in_red[qr + 5]])) > 1e-3


@pytest.mark.parametrize("geom", [(16, 64, 64), (32, 128, 128)])
def test_fp8_online_skipping_is_the_online_schedule_over_the_kept_keys(geom):
    # the online schedule with blocks of kb keys: dropping the whole block 2
    # leaves the same blocks as removing its tokens
    qr, kb, tile = geom
    q, k, v, cu, scale = _skip_case(kb, qr, seed=1)
    L = q.shape[0]
    counts = []
    o, lse, _ = oracle.varlen_attn_fp8_online(q, k, v, cu, scale, kblock=kb, threshold=8.0, tau=10.0,
                                              skip_block=(qr, kb), skip_tile_rows=tile, counts_out=counts)
    assert counts == [(L // qr - 1, math.ceil(L / tile) - 1)]
    full, _, _ = oracle.varlen_attn_fp8_online(q, k, v, cu, scale, kblock=kb, threshold=8.0)
    keep = np.r_[0:2 * kb, 3 * kb:L]
    red, _, _ = oracle.varlen_attn_fp8_online(q[keep], k[keep], v[keep], np.array([0, len(keep)], np.int32), scale,
                                              kblock=kb, threshold=8.0)
    pos_in_red = {int(t): i for i, t in enumerate(keep)}
    for t in range(L):
        if qr <= t < 2 * qr:
            np.testing.assert_allclose(o[t], full[t], rtol=0, atol=1e-12)
        elif t in pos_in_red:
            np.testing.assert_allclose(o[t], red[pos_in_red[t]], rtol=0, atol=1e-12)


def test_fp8_huge_threshold_skips_nothing():
    g = np.random.default_rng(14)
    T, H, D = 700, 2, 32
    q, k, v = (g.standard_normal((T, H, D)) * 2 for _ in range(3))
    cu = np.array([0, 300, 300, 700], np.int32)
    for fn, kw in ((oracle.varlen_attn_fp8, {}), (oracle.varlen_attn_fp8_online, {"kblock": 128, "threshold": 8.0})):
        counts = []
        o, lse, _ = fn(q, k, v, cu, 0.2, tau=1e30, skip_block=(32, 128), skip_tile_rows=128, counts_out=counts, **kw)
        o0, l0, _ = fn(q, k, v, cu, 0.2, **kw)
        assert counts == [(0, 0)]
        assert np.array_equal(o, o0) and np.array_equal(lse, l0)
    with pytest.raises(ValueError):
        oracle.varlen_attn_fp8(q, k, v, cu, 0.2, tau=4.0)  # a finite tau needs the block geometry


def test_fp8_skipping_sampled_rows_equal_full_evaluation():
    q, k, v, cu, scale = _skip_case(64, 16, seed=2)
    o, lse, _ = oracle.varlen_attn_fp8(q, k, v, cu, scale, tau=10.0, skip_block=(16, 64), skip_tile_rows=64)
    rows = np.array([0, 15, 16, 21, 31, 32, 150, 255], np.int32)
    o2, l2, _ = oracle.varlen_attn_fp8(q, k, v, cu, scale, tau=10.0, skip_block=(16, 64), skip_tile_rows=64,
                                       rows=rows)
    assert np.array_equal(o2, o[rows]) and np.array_equal(l2, lse[rows])


# ----------------------------------------------- Q/K prologue with e4m3 output (bound scale)

def test_fp8_prologue_scale_is_the_normalised_rows_bound():
    # deq = sqrt(D) * max |w| / 448 in float arithmetic, whatever the data
    g = np.random.default_rng(20)
    for D in (64, 128):
        w = g.uniform(0.5, 1.5, D)
        w[3] = -1.75  # the largest magnitude is negative
        x = g.standard_normal((50, 2, D))
        _, deq = oracle.qk_norm_rope_e4m3(x, w, np.arange(50, dtype=np.int32), 1e-6, 10000.0)
        amax = np.float32(np.sqrt(np.float32(D))) * np.float32(1.75)
        assert deq == np.float32(amax / np.float32(448.0))
        _, deq2 = oracle.qk_norm_rope_e4m3(x * 100.0, w, np.arange(50, dtype=np.int32), 1e-6, 10000.0)
        assert deq2 == deq


def test_fp8_prologue_one_hot_row_reaches_the_bound():
    # x = (a, 0, ..., 0) at position 0: the normalised row is sqrt(D) at d = 0,
    # times w_0 = max |w|, i.e. exactly the bound: code +-448 (0x7E / 0xFE),
    # every other element 0
    D = 128
    w = np.full(D, 0.75)
    w[0] = 1.25
    x = np.zeros((2, 1, D))
    x[0, 0, 0] = 1000.0
    x[1, 0, 0] = -1000.0
    codes, _ = oracle.qk_norm_rope_e4m3(x, w, np.zeros(2, np.int32), 1e-12, 10000.0)
    assert codes[0, 0, 0] == 0x7E and codes[1, 0, 0] == 0xFE
    assert np.all(codes[:, 0, 1:] == 0)


def test_fp8_prologue_codes_are_within_an_e4m3_step_of_the_rotated_rows():
    g = np.random.default_rng(21)
    T, H, D = 300, 3, 128
    x = g.standard_normal((T, H, D))
    x[7] *= 40.0
    w = g.uniform(0.5, 1.5, D)
    pos = g.integers(0, 60000, T).astype(np.int32)
    for style in (oracle.ROPE_INTERLEAVED, oracle.ROPE_HALF):
        codes, deq = oracle.qk_norm_rope_e4m3(x, w, pos, 1e-6, 10000.0, style)
        y = oracle.qk_norm_rope(x, w, pos, 1e-6, 10000.0, style)
        back = _decode(codes) * float(deq)
        assert np.all(np.abs(y) <= 448.0 * float(deq) * (1 + 1e-6))  # the bound holds
        assert np.all(np.abs(back - y) <= np.maximum(2.0 ** -4 * np.abs(y), 2.0 ** -10 * float(deq)) * (1 + 1e-6))
        # sampled rows = full evaluation
        rows = np.array([0, 7, 150, 299], np.int32)
        c2, d2 = oracle.qk_norm_rope_e4m3(x, w, pos, 1e-6, 10000.0, style, rows=rows)
        assert np.array_equal(c2, codes[rows]) and d2 == deq
