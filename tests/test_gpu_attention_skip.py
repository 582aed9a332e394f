"""GPU parity of pqk_varlen_attn_fwd_skip (key-block skipping) against the
float64 oracle.

"Skip-Softmax" leaves out the softmax and P x V work of unimportant blocks
("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长", bullet on TRTLLM_ATTN
SAGE and Skip-Softmax). The kernel takes each block decision in fp32 on the
tensor-core scores, the oracle in float64, so every case here first checks
(in float64, from the inputs alone) which decisions lie within MARGIN of the
threshold. Where none does, the decisions are the same on both sides: the
outputs are compared with the attention tolerances and the skip counts
exactly. Rows of a block with such a decision may differ from the oracle by
at most twice the softmax share of the undecided key blocks times max|V|.
"""

import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import (LSE_MAX_ABS, SKIP_BLOCK, SKIP_TILE_ROWS, assert_attention, bf16_to_f64, max_abs, to_dev,
                             to_dev_bf16, torch_cuda)

pytestmark = pytest.mark.gpu

# log2 units. An fp32 dot product of 128 bf16 pairs is within 128 * 2^-24 *
# sum |q_d k_d| of the exact one; with |q| |k| <= ~1000 here and the scale
# 1/sqrt(128), that is < 1e-3 in log2 units, so 0.02 leaves a factor of 20.
MARGIN = 0.02


def decision_margins(x, tau, scale, blocks=None, per_block=False):
    """Smallest |max_rows(tile max - earlier max) + tau| over the checked
    (request, head, 32-row block, key block >= 1) decisions, in float64.
    blocks: None (all) or a set of (request, 32-row block index). With
    per_block, a dict {(request, block, head): margins of key blocks 1..}."""
    q, k = (wl.bf16_bits_to_f64(x[n]) if x[n].dtype == np.uint16 else x[n] for n in ("q", "k"))
    cu = x["cu_seqlens"]
    H = q.shape[1]
    worst = math.inf
    by_block = {}
    for i in range(len(cu) - 1):
        lo, hi = int(cu[i]), int(cu[i + 1])
        L = hi - lo
        if L == 0:
            continue
        nkb = (L + 127) // 128
        for b in range((L + 31) // 32):
            if blocks is not None and (i, b) not in blocks:
                continue
            r0, r1 = lo + 32 * b, min(hi, lo + 32 * b + 32)
            for h in range(H):
                u = scale * (q[r0:r1, h] @ k[lo:hi, h].T) / math.log(2.0)
                pad = np.full((r1 - r0, nkb * 128), -np.inf)
                pad[:, :L] = u
                tmax = pad.reshape(r1 - r0, nkb, 128).max(axis=2)
                prev = np.maximum.accumulate(tmax, axis=1)[:, :-1]
                d = (tmax[:, 1:] - prev + tau).max(axis=0)
                by_block[(i, b, h)] = np.abs(d)
                if d.size:
                    worst = min(worst, float(np.abs(d).min()))
    return by_block if per_block else worst


def run_skip(x, tau, scale, counts=True):
    torch = torch_cuda()
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    cu = to_dev(x["cu_seqlens"])
    c = torch.zeros(2, dtype=torch.int64, device="cuda") if counts else None
    o, lse = pqk.varlen_attn_fwd_skip(q, k, v, cu, tau, softmax_scale=scale, want_lse=True, skip_counts=c)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    return o, lse, (tuple(int(a) for a in c.cpu()) if counts else None)


@pytest.mark.parametrize("lens, H, D", [([4096], 16, 128), ([300, 0, 513, 1], 2, 64), ([255, 256, 257], 3, 128)])
def test_infinite_threshold_is_bitwise_the_plain_kernel(lens, H, D):
    torch = torch_cuda()
    w = wl.custom(lens, H, D, seed=sum(lens))
    x = wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(D)
    o, lse, counts = run_skip(x, math.inf, scale)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    o2, lse2 = pqk.varlen_attn_fwd(q, k, v, to_dev(x["cu_seqlens"]), softmax_scale=scale, want_lse=True)
    torch.cuda.synchronize()
    assert counts == (0, 0)
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(lse, lse2)


@pytest.mark.parametrize("lens, H, D, seed", [([700, 1300, 129], 2, 128, 24), ([1000, 37, 640], 3, 64, 8),
                                              ([2048], 2, 128, 9), ([640, 0, 257, 1], 2, 128, 44)])
@pytest.mark.parametrize("tau", [4.0, 8.0])
def test_block_scaled_matches_oracle_and_counts(lens, H, D, seed, tau):
    w = wl.custom(lens, H, D, seed=seed)
    x = wl.block_scaled_attention_inputs(w)
    scale = 1.0 / math.sqrt(D)
    assert decision_margins(x, tau, scale) >= MARGIN
    o, lse, counts = run_skip(x, tau, scale)
    ro, rl, rc = oracle.varlen_attn_skip(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, tau, block=SKIP_BLOCK,
                                        tile_rows=SKIP_TILE_ROWS)
    assert rc[0] > 0, "the case must drop some blocks"
    assert counts == rc
    assert_attention(bf16_to_f64(o), ro, f"{lens} H{H} D{D} tau {tau}", peaked=True)
    lse = lse.cpu().numpy().astype(np.float64).T
    assert max_abs(lse, rl) <= LSE_MAX_ABS


def test_skip_kernel_is_deterministic():
    torch = torch_cuda()
    w = wl.custom([700, 1300, 129], 2, 128, seed=24)
    x = wl.block_scaled_attention_inputs(w)
    runs = [run_skip(x, 8.0, 1.0 / math.sqrt(128)) for _ in range(3)]
    for o, lse, c in runs[1:]:
        assert torch.equal(o.view(torch.int16), runs[0][0].view(torch.int16))
        assert torch.equal(lse, runs[0][1]) and c == runs[0][2]


def test_local_inputs_sampled_rows():
    # the stand-in for video attention (weight on nearby (t, h, w) ids) at
    # 16,384 tokens, on sampled rows. Scores vary continuously here, so a few
    # blocks have a decision within MARGIN of the threshold, which fp32 and
    # float64 may take differently; their rows get the bound of either choice.
    w = wl.custom([16384], 4, 128, seed=11)
    x = wl.local_attention_inputs(w, amplitude=16.0)
    H, scale, tau = 4, 1.0 / math.sqrt(128), 8.0
    rows = wl.sample_rows(w, per_segment=48)
    margins = decision_margins(x, tau, scale, {(0, int(r) // 32) for r in rows}, per_block=True)
    o, lse, counts = run_skip(x, tau, scale)
    assert counts[0] > 0
    o = bf16_to_f64(o)[rows]
    lse = lse.cpu().numpy().astype(np.float64).T[rows]
    ro, rl, _ = oracle.varlen_attn_skip(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, tau, block=SKIP_BLOCK,
                                       tile_rows=SKIP_TILE_ROWS, rows=rows)
    q, k = wl.bf16_bits_to_f64(x["q"]), wl.bf16_bits_to_f64(x["k"])
    vmax = float(np.abs(wl.bf16_bits_to_f64(x["v"])).max())
    n_clear = 0
    for n, r in enumerate(rows):
        for h in range(H):
            undecided = np.nonzero(margins[(0, int(r) // 32, h)] < MARGIN)[0] + 1
            if undecided.size == 0:
                n_clear += 1
                assert_attention(o[n, h], ro[n, h], f"local row {r} head {h}", peaked=True)
                assert abs(lse[n, h] - rl[n, h]) <= LSE_MAX_ABS
                continue
            s_row = scale * (k[:, h] @ q[r, h])
            p = np.exp(s_row - s_row.max())
            share = sum(p[128 * j:128 * (j + 1)].sum() for j in undecided) / p.sum()
            assert max_abs(o[n, h], ro[n, h]) <= 2.0 * share * vmax + 2e-2
    assert n_clear >= len(rows) * H // 2


def test_local_inputs_58048_tokens_sampled_rows():
    # the bench's block-skipping workload (local stand-in at 58,048 tokens,
    # 24 heads, tau = 8) on 12 sampled rows: decided (row, head) pairs
    # against the oracle, the others within the bound of either choice
    w = wl.config(3)
    x = wl.local_attention_inputs(w, amplitude=16.0)
    scale, tau = 1.0 / math.sqrt(128), 8.0
    rows = wl.sample_rows(w, per_segment=12)
    margins = decision_margins(x, tau, scale, {(0, int(r) // 32) for r in rows}, per_block=True)
    o, lse, counts = run_skip(x, tau, scale)
    assert counts[0] > 0
    o = bf16_to_f64(o)[rows]
    ro, rl, _ = oracle.varlen_attn_skip(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, tau, block=SKIP_BLOCK,
                                       tile_rows=SKIP_TILE_ROWS, rows=rows)
    q, k = wl.bf16_bits_to_f64(x["q"]), wl.bf16_bits_to_f64(x["k"])
    vmax = float(np.abs(wl.bf16_bits_to_f64(x["v"])).max())
    n_clear = 0
    for n, r in enumerate(rows):
        for h in range(w.H):
            undecided = np.nonzero(margins[(0, int(r) // 32, h)] < MARGIN)[0] + 1
            if undecided.size == 0:
                n_clear += 1
                assert_attention(o[n, h], ro[n, h], f"local 58k row {r} head {h}", peaked=True)
                continue
            s_row = scale * (k[:, h] @ q[r, h])
            p = np.exp(s_row - s_row.max())
            share = sum(p[128 * j:128 * (j + 1)].sum() for j in undecided) / p.sum()
            assert max_abs(o[n, h], ro[n, h]) <= 2.0 * share * vmax + 2e-2
    assert n_clear >= len(rows) * w.H // 8
