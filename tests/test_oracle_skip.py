"""Pins for the oracle's attention with key-block skipping (CPU only).

"Skip-Softmax" skips the softmax and P x V work of unimportant blocks ("FastH3
在八卡 B300 上实现完整 MP4 生成快于播放时长", bullet on TRTLLM_ATTN SAGE and
Skip-Softmax; "MiniMax H3 FastH3 real-time serving with vLLM-Omni", bullet
"Sparse & quantized attention"). The block rule is a reading: for a block of
qrows query rows x kblock keys, key block j >= 1 is dropped when every row's
block maximum of score / ln 2 lies more than tau below its maximum over the
earlier blocks. The pages give no block size, so the oracle takes the geometry
as an argument; every pin below runs at several geometries, among them ones
no kernel here uses (16 x 64, 8 x 48), so that the rule is checked apart from
any one tile shape. The pins check it against facts that do not come from the
oracle: the plain attention when nothing can be skipped, a dense brute force
over the kept keys in constructed cases whose decisions are forced, the error
bound of dropping keys whose weights are below 2^-tau, and monotonicity in
tau.
"""

import math

import numpy as np
import pytest

from oracle import oracle
from tests.bruteforce import padded_masked_attention


# (query rows, keys, tile rows): two geometries no kernel here uses, then the
# attention kernel's softmax warp x K/V tile with its 128-row query tile
GEOMETRIES = [(16, 64, 64), (8, 48, 24), (32, 128, 128)]


def _skip(q, k, v, cu, scale, tau, geom, rows=None):
    qr, kb, tile = geom
    return oracle.varlen_attn_skip(q, k, v, cu, scale, tau, block=(qr, kb), tile_rows=tile, rows=rows)


def _softmax_subset(q_row, k, v, keep_keys, scale):
    """Dense softmax attention of one query row over the listed key rows."""
    s = scale * (k[keep_keys] @ q_row)
    m = s.max()
    p = np.exp(s - m)
    return (p[:, None] * v[keep_keys]).sum(axis=0) / p.sum(), m + math.log(p.sum())


@pytest.mark.parametrize("geom", GEOMETRIES)
@pytest.mark.parametrize("lens", [[1], [129], [300], [5, 0, 257, 1], [640]])
def test_large_tau_is_plain_attention(lens, geom):
    H, D = 2, 16
    T = sum(lens)
    g = np.random.default_rng(T)
    q, k, v = (g.standard_normal((T, H, D)) * 3 for _ in range(3))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    scale = 1.0 / math.sqrt(D)
    o, lse, counts = _skip(q, k, v, cu, scale, 1e30, geom)
    ob, lb = padded_masked_attention(q, k, v, cu, scale)
    assert counts == (0, 0)
    assert np.max(np.abs(o - ob)) <= 1e-12
    assert np.max(np.abs(lse - lb)) <= 1e-12


def _constructed(geom, seed=0):
    """One request of four key blocks, one head, D = 16. Every query is close
    to +a*u; keys of key block 2 are close to -a*u, so block 2's scores lie far
    below the earlier blocks' and it is dropped, except for query block 1,
    which holds row qrows + 5 whose query points at block 2's keys. Keys of
    block 0 are also close to -a*u but block 0 is never dropped."""
    qr, kb, _ = geom
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
    return q[:, None, :], k[:, None, :], v[:, None, :], np.array([0, L], np.int32), 1.0 / math.sqrt(D)


@pytest.mark.parametrize("geom", GEOMETRIES)
def test_forced_decisions_match_bruteforce_over_kept_keys(geom):
    qr, kb, tile = geom
    q, k, v, cu, scale = _constructed(geom)
    tau = 10.0
    o, lse, counts = _skip(q, k, v, cu, scale, tau, geom)
    L = q.shape[0]
    all_keys = np.arange(L)
    without_block2 = np.concatenate([np.arange(0, 2 * kb), np.arange(3 * kb, L)])
    for r in range(L):
        keep = all_keys if qr <= r < 2 * qr else without_block2
        ob, lb = _softmax_subset(q[r, 0], k[:, 0], v[:, 0], keep, scale)
        np.testing.assert_allclose(o[r, 0], ob, rtol=0, atol=1e-12)
        assert abs(lse[r, 0] - lb) <= 1e-12
    # every query block but one drops key block 2; so does every tile but the
    # one holding query block 1
    assert counts == (L // qr - 1, math.ceil(L / tile) - 1)
    # row qrows + 5 attends mostly to block 2: dropping it would change its output a lot
    o_plain, _ = oracle.varlen_attn(q, k, v, cu, scale)
    assert np.max(np.abs(o[qr + 5] - o_plain[qr + 5])) <= 1e-12


@pytest.mark.parametrize("geom", GEOMETRIES)
def test_very_negative_tau_keeps_only_the_first_key_block(geom):
    qr, kb, tile = geom
    g = np.random.default_rng(5)
    L, D = 300, 8
    q, k, v = (g.standard_normal((L, 1, D)) for _ in range(3))
    cu = np.array([0, L], np.int32)
    scale = 0.4
    o, _, counts = _skip(q, k, v, cu, scale, -1e30, geom)
    for r in range(L):
        ob, _ = _softmax_subset(q[r, 0], k[:, 0], v[:, 0], np.arange(kb), scale)
        np.testing.assert_allclose(o[r, 0], ob, rtol=0, atol=1e-12)
    nqb, ntile, nkb = math.ceil(L / qr), math.ceil(L / tile), math.ceil(L / kb)
    assert counts == (nqb * (nkb - 1), ntile * (nkb - 1))


def _block_scales(g, L, kb):
    """Per-key scale, constant over each block of kb keys: 3 for block 0, else
    drawn from [0.05, 3], so that some blocks' scores are far below others'."""
    nb = math.ceil(L / kb)
    s = np.concatenate([[3.0], g.uniform(0.05, 3.0, nb - 1)])
    return np.repeat(s, kb)[:L, None, None]


@pytest.mark.parametrize("geom", GEOMETRIES)
def test_error_bound_of_dropped_keys(geom):
    # peaked scores so that blocks are dropped at tau = 6: every dropped key has
    # weight < 2^-tau of the row maximum, so the dropped share of the softmax
    # mass is below n_dropped * 2^-tau and the output moves by at most twice that
    # share times max |v|
    g = np.random.default_rng(11)
    L, H, D = 700, 2, 32
    q = g.standard_normal((L, H, D)) * 2.5
    k = g.standard_normal((L, H, D)) * _block_scales(g, L, geom[1])
    v = g.standard_normal((L, H, D))
    cu = np.array([0, L], np.int32)
    scale = 1.0 / math.sqrt(D)
    tau = 6.0
    o, _, counts = _skip(q, k, v, cu, scale, tau, geom)
    assert counts[0] > 0
    ob, _ = oracle.varlen_attn(q, k, v, cu, scale)
    bound = 2.0 * L * 2.0 ** -tau * np.abs(v).max()
    assert np.max(np.abs(o - ob)) <= bound
    assert np.max(np.abs(o - ob)) > 0.0


@pytest.mark.parametrize("geom", GEOMETRIES)
def test_fewer_skips_as_tau_grows(geom):
    g = np.random.default_rng(3)
    L, H, D = 900, 2, 32
    q = g.standard_normal((L, H, D)) * 2.5
    k = g.standard_normal((L, H, D)) * _block_scales(g, L, geom[1])
    v = g.standard_normal((L, H, D))
    cu = np.array([0, 400, L], np.int32)
    prev = None
    for tau in (0.0, 2.0, 4.0, 8.0, 16.0):
        _, _, counts = _skip(q, k, v, cu, 1.0 / math.sqrt(D), tau, geom)
        assert counts[1] <= counts[0]
        if prev is not None:
            assert counts[0] <= prev[0] and counts[1] <= prev[1]
        prev = counts


@pytest.mark.parametrize("geom", GEOMETRIES)
def test_sampled_rows_equal_full_evaluation(geom):
    qr = geom[0]
    q, k, v, cu, scale = _constructed(geom, 1)
    o, lse, _ = _skip(q, k, v, cu, scale, 10.0, geom)
    L = q.shape[0]
    rows = np.array([0, qr - 1, qr, qr + 5, 2 * qr - 1, 2 * qr, L // 2 + 3, L - 1], np.int32)
    os_, ls, counts = _skip(q, k, v, cu, scale, 10.0, geom, rows=rows)
    assert counts is None
    assert np.array_equal(os_, o[rows]) and np.array_equal(ls, lse[rows])


@pytest.mark.parametrize("geom", GEOMETRIES)
@pytest.mark.parametrize("tau, skipped", [(11.0, True), (11.6, False), (12.0, False)])
def test_threshold_is_in_log2_units(tau, skipped, geom):
    # scores (scale 1, D = 1): one key of block 0 scores 8, every other key 0.
    # Block 1's maximum lies 8 nats = 8 / ln 2 = 11.54 bits below block 0's, so
    # block 1 is dropped exactly when tau < 11.54
    qr, kb, tile = geom
    L = kb + kb * 9 // 16  # two key blocks, the second partial
    first_v = kb + kb * 11 // 64
    q = np.ones((L, 1, 1))
    k = np.zeros((L, 1, 1))
    k[5] = 8.0
    v = np.zeros((L, 1, 1))
    v[first_v:] = 1.0  # block 1 carries all of the value mass
    cu = np.array([0, L], np.int32)
    o, _, counts = _skip(q, k, v, cu, 1.0, tau, geom)
    expect_block1 = 0.0 if skipped else (L - first_v) / (math.exp(8.0) + (L - 1))
    assert counts == ((math.ceil(L / qr), math.ceil(L / tile)) if skipped else (0, 0))
    np.testing.assert_allclose(o[:, 0, 0], expect_block1, rtol=1e-12, atol=0)


def test_geometry_is_validated():
    q = np.zeros((10, 1, 4))
    cu = np.array([0, 10], np.int32)
    for qr, kb, tile in [(0, 64, 64), (16, 0, 64), (16, 64, 24), (16, 64, 0)]:
        with pytest.raises(ValueError):
            _skip(q, q, q, cu, 1.0, 4.0, (qr, kb, tile))
