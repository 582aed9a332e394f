"""GPU parity of the FP8 (e4m3) Q/K quantisation and of the attention with
Q K^T on the FP8 tensor cores, against the float64 oracle.

SAGE quantises the attention computation to FP8 ("FastH3 在八卡 B300 上实现
完整 MP4 生成快于播放时长", bullet on TRTLLM_ATTN SAGE and Skip-Softmax). The
quantisation is integer (byte) work and must match the oracle bit for bit,
its scales exactly; the attention is compared with the attention tolerances
against the oracle's attention on the same quantised Q and K.
"""

import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import (ATTN_MAX_ABS, ATTN_REL_L2, ELEM_UNIT_MAX, LSE_MAX_ABS, SKIP_BLOCK, SKIP_TILE_ROWS,
                             assert_attention, bf16_to_f64, max_abs, rel_l2, to_dev, to_dev_bf16, torch_cuda)

pytestmark = pytest.mark.gpu


def _quantise_gpu(x, stride_pad=0):
    torch = torch_cuda()
    T, H, D = x["q"].shape
    if stride_pad:
        # Q and K as views into a wider fused row, as a QKV projection would give
        buf = torch.zeros((T, 2 * H * D + stride_pad), dtype=torch.bfloat16, device="cuda")
        buf[:, :H * D] = to_dev_bf16(x["q"]).view(T, H * D)
        buf[:, H * D + stride_pad // 2: 2 * H * D + stride_pad // 2] = to_dev_bf16(x["k"]).view(T, H * D)
        q = buf[:, :H * D].view(T, H, D)
        k = buf[:, H * D + stride_pad // 2: 2 * H * D + stride_pad // 2].view(T, H, D)
    else:
        q, k = to_dev_bf16(x["q"]), to_dev_bf16(x["k"])
    q8, k8, deq = pqk.quantize_qk_e4m3(q, k)
    torch.cuda.synchronize()
    return q8, k8, deq


@pytest.mark.parametrize("lens, H, D, pad", [([4096], 16, 128, 0), ([300, 0, 513, 1], 3, 128, 64),
                                             ([200, 312], 4, 64, 0), ([1], 1, 128, 0)])
def test_quantisation_is_bitwise_the_oracle(lens, H, D, pad):
    w = wl.custom(lens, H, D, seed=sum(lens) + H)
    x = wl.attention_inputs(w)
    q8, k8, deq = _quantise_gpu(x, pad)
    rq, rdq = oracle.quantize_e4m3(x["q"])
    rk, rdk = oracle.quantize_e4m3(x["k"])
    assert np.array_equal(q8.cpu().numpy(), rq)
    assert np.array_equal(k8.cpu().numpy(), rk)
    assert np.array_equal(deq.cpu().numpy(), np.concatenate([rdq, rdk]))


def test_quantisation_of_outliers_and_a_zero_head():
    w = wl.custom([3000], 4, 128, seed=5)
    x = wl.attention_inputs(w, outliers=True)
    q = wl.bf16_bits_to_f32(x["q"])
    q[:, 2] = 0.0
    x["q"] = wl.f32_to_bf16_bits(q)
    q8, k8, deq = _quantise_gpu(x)
    rq, rdq = oracle.quantize_e4m3(x["q"])
    rk, rdk = oracle.quantize_e4m3(x["k"])
    assert np.array_equal(q8.cpu().numpy(), rq) and np.array_equal(k8.cpu().numpy(), rk)
    assert np.array_equal(deq.cpu().numpy(), np.concatenate([rdq, rdk]))
    assert deq.cpu().numpy()[2] == 1.0


def _attn_gpu(x, scale):
    torch = torch_cuda()
    q8, k8, deq = _quantise_gpu(x)
    o, lse = pqk.varlen_attn_fwd_fp8qk(q8, k8, to_dev_bf16(x["v"]), deq, to_dev(x["cu_seqlens"]),
                                       softmax_scale=scale, want_lse=True)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    return o, lse


@pytest.mark.parametrize("lens", [[1], [127], [129], [255, 256, 257], [300, 0, 513, 1], [0, 0, 700],
                                  [384, 17, 2, 640]])
def test_attention_full(lens):
    H, D = 3, 128
    w = wl.custom(lens, H, D, seed=sum(lens) + 17)
    x = wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(D)
    o, lse = _attn_gpu(x, scale)
    ro, rl, _, _, _ = oracle.varlen_attn_fp8qk(x["q"], x["k"], x["v"], x["cu_seqlens"], scale)
    assert_attention(bf16_to_f64(o), ro, f"fp8 {lens}")
    assert max_abs(lse.cpu().numpy().astype(np.float64).T, rl) <= LSE_MAX_ABS


def test_attention_peaked_full():
    # Q x 8: each row's weight concentrates on few keys, where the FP8 score
    # error matters most
    H, D = 2, 128
    w = wl.custom([700, 1300], H, D, seed=23)
    x = wl.attention_inputs(w)
    x["q"] = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(x["q"]) * np.float32(8.0))
    scale = 1.0 / math.sqrt(D)
    o, lse = _attn_gpu(x, scale)
    ro, rl, _, _, _ = oracle.varlen_attn_fp8qk(x["q"], x["k"], x["v"], x["cu_seqlens"], scale)
    assert_attention(bf16_to_f64(o), ro, "fp8 peaked", peaked=True)
    assert max_abs(lse.cpu().numpy().astype(np.float64).T, rl) <= LSE_MAX_ABS


def test_attention_4096_tokens_full_and_error_against_bf16():
    w = wl.config(2)
    x = wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(w.D)
    o, lse = _attn_gpu(x, scale)
    ro, rl, _, _, _ = oracle.varlen_attn_fp8qk(x["q"], x["k"], x["v"], x["cu_seqlens"], scale)
    g = bf16_to_f64(o)
    assert_attention(g, ro, "fp8 4096 tokens")
    assert max_abs(lse.cpu().numpy().astype(np.float64).T, rl) <= LSE_MAX_ABS
    # the quantisation's own effect, against the unquantised oracle: small but present
    po, _ = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], scale)
    assert 1e-4 < rel_l2(ro, po) < 0.1


def test_attention_16k_sampled_rows():
    w = wl.custom([16384], 8, 128, seed=29)
    x = wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(128)
    rows = wl.sample_rows(w, per_segment=128)
    o, lse = _attn_gpu(x, scale)
    ro, rl, _, _, _ = oracle.varlen_attn_fp8qk(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, rows=rows)
    assert_attention(bf16_to_f64(o)[rows], ro, "fp8 16k sampled")
    assert max_abs(lse.cpu().numpy().astype(np.float64).T[rows], rl) <= LSE_MAX_ABS


def test_fp8_attention_is_deterministic():
    torch = torch_cuda()
    w = wl.custom([1000, 2000], 4, 128, seed=31)
    x = wl.attention_inputs(w)
    a = [_attn_gpu(x, 0.1) for _ in range(3)]
    for o, lse in a[1:]:
        assert torch.equal(o.view(torch.int16), a[0][0].view(torch.int16)) and torch.equal(lse, a[0][1])


@pytest.mark.parametrize("tau", [4.0, 8.0])
def test_fp8_with_block_skipping_matches_oracle_and_counts(tau):
    # decisions taken on the FP8 scores: margins checked on the dequantised
    # Q, K in float64, then outputs and skip counts against the oracle
    import torch
    from tests.test_gpu_attention_skip import MARGIN, decision_margins
    torch_cuda()
    w = wl.custom([700, 1300, 129], 2, 128, seed=24)
    x = wl.block_scaled_attention_inputs(w)
    scale = 1.0 / math.sqrt(128)
    counts = []
    ro, rl, q8r, k8r, deqr = oracle.varlen_attn_fp8qk(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, tau=tau,
                                                      skip_block=SKIP_BLOCK, skip_tile_rows=SKIP_TILE_ROWS,
                                                      counts_out=counts)
    H = w.H
    dec = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    xd = {"q": dec(q8r) * deqr[None, :H, None], "k": dec(k8r) * deqr[None, H:, None], "cu_seqlens": x["cu_seqlens"]}
    assert decision_margins(xd, tau, scale) >= MARGIN
    q8, k8, deq = _quantise_gpu(x)
    c = torch.zeros(2, dtype=torch.int64, device="cuda")
    o, lse = pqk.varlen_attn_fwd_fp8qk(q8, k8, to_dev_bf16(x["v"]), deq, to_dev(x["cu_seqlens"]), softmax_scale=scale,
                                       want_lse=True, skip_threshold_log2=tau, skip_counts=c)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    assert tuple(int(a) for a in c.cpu()) == counts[0] and counts[0][0] > 0
    assert_attention(bf16_to_f64(o), ro, f"fp8 + skip tau {tau}", peaked=True)
    assert max_abs(lse.cpu().numpy().astype(np.float64).T, rl) <= LSE_MAX_ABS


def test_joint_sequence_58048_sampled():
    # the bench's workload and launch configuration, on 96 sampled rows
    w = wl.config(3)
    x = wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(w.D)
    rows = wl.sample_rows(w, per_segment=96)
    o, lse = _attn_gpu(x, scale)
    ro, rl, _, _, _ = oracle.varlen_attn_fp8qk(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, rows=rows)
    assert_attention(bf16_to_f64(o)[rows], ro, "fp8 58,048 tokens sampled")
    assert max_abs(lse.cpu().numpy().astype(np.float64).T[rows], rl) <= LSE_MAX_ABS


# ---------------------------------------------------------------- Q, K, V and P in FP8

def _full_fp8_gpu(x, scale, tau=math.inf):
    torch = torch_cuda()
    q8, k8, deq_qk = _quantise_gpu(x)
    v8, deq_v = pqk.quantize_e4m3(to_dev_bf16(x["v"]))
    deq = torch.cat([deq_qk, deq_v]).contiguous()
    c = torch.zeros(2, dtype=torch.int64, device="cuda")
    o, lse = pqk.varlen_attn_fwd_fp8(q8, k8, v8, deq, to_dev(x["cu_seqlens"]), softmax_scale=scale, want_lse=True,
                                     skip_threshold_log2=tau, skip_counts=c)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    return o, lse, v8, deq, tuple(int(a) for a in c.cpu())


# The whole-FP8 kernel is an online softmax over K/V tiles of 128 keys whose
# running maximum (log2 units) is set by the first tile and moves only when a
# tile's maximum exceeds it by more than 8: its rounding schedule for P.
KERNEL_KBLOCK, KERNEL_THRESHOLD = 128, 8.0


def _decode(c):
    import torch
    return torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def _e4m3_quantum(p):
    """Spacing of the e4m3 grid at p > 0: 2^(e - 3) in the normal range, 2^-9 below 2^-6."""
    e = np.floor(np.log2(np.maximum(p, 2.0 ** -6)))
    return np.exp2(e - 3)


def _kept_keys(qd, kd, scale, lo, hi, t, h, tau):
    """Keys of row t's request kept by the block-skipping rule (32-row query
    blocks x 128-key blocks counted from the request's first token, decided
    in float64 on the dequantised scores); all of them for tau = inf."""
    L = hi - lo
    if math.isinf(tau):
        return np.ones(L, bool)
    qr, kb = SKIP_BLOCK
    r0 = lo + (t - lo) // qr * qr
    r1 = min(hi, r0 + qr)
    u = scale * (qd[r0:r1, h] @ kd[lo:hi, h].T) / math.log(2.0)
    nkb = (L + kb - 1) // kb
    pad = np.full((r1 - r0, nkb * kb), -np.inf)
    pad[:, :L] = u
    tmax = pad.reshape(r1 - r0, nkb, kb).max(axis=2)
    prev = np.maximum.accumulate(tmax, axis=1)
    drop = np.zeros(nkb, bool)
    drop[1:] = np.all(tmax[:, 1:] < prev[:, :-1] - tau, axis=0)
    return np.repeat(~drop, kb)[:L]


def _row_terms(qd, kd, scale, lo, hi, t, h, keep):
    """For row t, head h over the kept keys of [lo, hi): the probabilities p_j
    against the maximum over those keys, and c_j = 2^(M - m_j), where m_j is
    the kernel's running maximum when key j's tile is visited (c_j >= 1;
    dropped tiles do not move it). p is 0 at dropped keys."""
    u = scale * (kd[lo:hi, h] @ qd[t, h]) / math.log(2.0)
    u = np.where(keep, u, -np.inf)
    M = u.max()
    m_at = np.empty_like(u)
    m = -np.inf
    for b0 in range(0, hi - lo, KERNEL_KBLOCK):
        bmax = u[b0:b0 + KERNEL_KBLOCK].max()
        if b0 == 0 or bmax > m + KERNEL_THRESHOLD:
            m = bmax
        m_at[b0:b0 + KERNEL_KBLOCK] = m
    return np.exp2(u - M), np.exp2(M - m_at)


def _check_full_fp8(x, scale, what, rows=None, peaked=False, tau=math.inf):
    """Element-wise against the oracle, twice.

    (1) The definition (oracle.varlen_attn_fp8: each probability p_j <= 1
    rounded to e4m3 against its row's exact maximum, the denominator
    unrounded). The kernel rounds each p against a running maximum that is
    never above the row's; e4m3 puts both roundings within max(2^-4 p_j,
    2^-10) of p_j (in units of the row's maximum), so each numerator term
    differs by at most max(2^-3 p_j, 2^-9) |v~_j| and each output element by
    at most the sum of those over the row's keys, divided by sum_j p_j. The
    test allows that row's sum plus the attention tolerance.

    (2) The kernel's own rounding schedule (oracle.varlen_attn_fp8_online with
    128-key blocks and threshold 8): the attention tolerances (relative L2 <=
    1e-2 over all elements; per element the max-abs bound, or on peaked
    inputs the unit-scale bound) plus, per row, one e4m3 step of each key
    whose probability lies within 2^-10 (relative) of an e4m3 rounding
    midpoint: the kernel rounds fp32 probabilities and the oracle float64
    ones, so only those keys can round differently.

    With a finite tau (block skipping) both sides drop the same key blocks
    (the callers check that no decision lies near the threshold), the sums
    run over the kept keys, and the skip counts must be equal."""
    o, lse, v8, deq, counts = _full_fp8_gpu(x, scale, tau)
    T, H, D = x["q"].shape
    sel = np.arange(T) if rows is None else rows
    kw = {} if math.isinf(tau) else {"tau": tau, "skip_block": SKIP_BLOCK, "skip_tile_rows": SKIP_TILE_ROWS}
    c_def, c_sch = [], []
    rd, rld, rdeq = oracle.varlen_attn_fp8(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, rows=rows,
                                           counts_out=c_def, **kw)
    rs, rls, _ = oracle.varlen_attn_fp8_online(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, kblock=KERNEL_KBLOCK,
                                               threshold=KERNEL_THRESHOLD, rows=rows, counts_out=c_sch, **kw)
    assert np.array_equal(deq.cpu().numpy(), rdeq)
    if math.isinf(tau):
        assert counts == (0, 0)
    elif rows is None:
        assert c_def == c_sch == [counts], f"{what}: skip counts {counts} vs oracle {c_def}"
    g = bf16_to_f64(o)[sel]
    assert rel_l2(g, rs) <= ATTN_REL_L2, f"{what}: rel-L2 {rel_l2(g, rs):.3e} against the kernel's schedule"
    qd, kd, vd = (_decode(c) * dq[None, :, None]
                  for c, dq in (oracle.quantize_e4m3(x[n]) for n in ("q", "k", "v")))
    cu = x["cu_seqlens"]
    for n, t in enumerate(sel):
        i = int(np.searchsorted(cu, t, side="right") - 1)
        lo, hi = int(cu[i]), int(cu[i + 1])
        for h in range(H):
            keep = _kept_keys(qd, kd, scale, lo, hi, t, h, tau)
            p, c = _row_terms(qd, kd, scale, lo, hi, t, h, keep)
            l = p.sum()
            av = np.abs(vd[lo:hi, h])
            # (1) the definition
            bound = ATTN_MAX_ABS + (np.where(keep, np.maximum(2.0 ** -3 * p, 2.0 ** -9), 0.0)[:, None] * av).sum(0) / l
            err = np.abs(g[n, h] - rd[n, h])
            assert np.all(err <= bound), f"{what}: row {t} head {h}: {err.max():.3e} over the definition's bound"
            # (2) the schedule: keys near a rounding midpoint, in the frame the kernel rounds in
            ps = p * c
            qn = _e4m3_quantum(np.where(keep, ps, 1.0))
            frac = ps / qn - np.floor(ps / qn)
            near = keep & (np.abs(frac - 0.5) * qn <= 2.0 ** -10 * ps)
            slack = (near[:, None] * (qn / c)[:, None] * av).sum(0) / l
            err = np.abs(g[n, h] - rs[n, h])
            tol = ELEM_UNIT_MAX * np.maximum(1.0, np.abs(rs[n, h])) if peaked else ATTN_MAX_ABS
            assert np.all(err <= tol + slack), f"{what}: row {t} head {h}: {err.max():.3e} against the schedule"
    assert max_abs(lse.cpu().numpy().astype(np.float64).T[sel], rls) <= LSE_MAX_ABS
    assert max_abs(rls, rld) <= 1e-9  # the lse does not depend on P's rounding


def test_v_quantisation_is_bitwise_the_oracle():
    torch = torch_cuda()
    w = wl.custom([300, 0, 513, 1], 3, 128, seed=41)
    x = wl.attention_inputs(w)
    v8, deq = pqk.quantize_e4m3(to_dev_bf16(x["v"]))
    torch.cuda.synchronize()
    rc, rd = oracle.quantize_e4m3(x["v"])
    assert np.array_equal(v8.cpu().numpy(), rc) and np.array_equal(deq.cpu().numpy(), rd)


@pytest.mark.parametrize("lens", [[1], [129], [255, 256, 257], [300, 0, 513, 1], [384, 17, 2, 640]])
def test_full_fp8_attention(lens):
    w = wl.custom(lens, 3, 128, seed=sum(lens) + 43)
    _check_full_fp8(wl.attention_inputs(w), 1.0 / math.sqrt(128), f"full fp8 {lens}")


def test_full_fp8_attention_peaked():
    w = wl.custom([700, 1300], 2, 128, seed=44)
    x = wl.attention_inputs(w)
    x["q"] = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(x["q"]) * np.float32(8.0))
    _check_full_fp8(x, 1.0 / math.sqrt(128), "full fp8 peaked", peaked=True)


def test_full_fp8_attention_16k_sampled_and_error_against_bf16():
    w = wl.custom([16384], 4, 128, seed=45)
    x = wl.attention_inputs(w)
    rows = wl.sample_rows(w, per_segment=64)
    _check_full_fp8(x, 1.0 / math.sqrt(128), "full fp8 16k", rows=rows)
    ro, _, _ = oracle.varlen_attn_fp8(x["q"], x["k"], x["v"], x["cu_seqlens"], 1.0 / math.sqrt(128), rows=rows)
    po, _ = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], 1.0 / math.sqrt(128), rows=rows)
    assert 1e-4 < rel_l2(ro, po) < 0.1


def test_full_fp8_attention_is_deterministic():
    torch = torch_cuda()
    w = wl.custom([1000, 2000], 4, 128, seed=46)
    x = wl.attention_inputs(w)
    a = [_full_fp8_gpu(x, 0.1) for _ in range(3)]
    for o, lse, _, _, _ in a[1:]:
        assert torch.equal(o.view(torch.int16), a[0][0].view(torch.int16)) and torch.equal(lse, a[0][1])


@pytest.mark.parametrize("lens, seed", [([700, 1300, 129], 47), ([640, 0, 257, 1], 48)])
@pytest.mark.parametrize("tau", [4.0, 8.0])
def test_full_fp8_with_block_skipping_matches_oracle_and_counts(lens, seed, tau):
    # SAGE FP8 with Skip-Softmax together: decisions taken on the FP8 scores
    # (margins checked on the dequantised Q, K in float64), then every element
    # against both oracles and the skip counts exactly
    import torch
    from tests.test_gpu_attention_skip import MARGIN, decision_margins
    torch_cuda()
    w = wl.custom(lens, 2, 128, seed=seed)
    x = wl.block_scaled_attention_inputs(w)
    scale = 1.0 / math.sqrt(128)
    H = w.H
    (q8r, dqr), (k8r, dkr) = oracle.quantize_e4m3(x["q"]), oracle.quantize_e4m3(x["k"])
    xd = {"q": _decode(q8r) * dqr[None, :, None], "k": _decode(k8r) * dkr[None, :, None],
          "cu_seqlens": x["cu_seqlens"]}
    assert decision_margins(xd, tau, scale) >= MARGIN
    _check_full_fp8(x, scale, f"full fp8 + skip tau {tau} {lens}", peaked=True, tau=tau)
    _, _, _, _, counts = _full_fp8_gpu(x, scale, tau)
    assert counts[0] > 0


def test_full_fp8_skipping_with_infinite_threshold_is_bitwise_the_plain_kernel():
    torch = torch_cuda()
    w = wl.custom([1000, 37, 640], 2, 128, seed=49)
    x = wl.attention_inputs(w)
    a = _full_fp8_gpu(x, 0.1)
    q8, k8, deq_qk = _quantise_gpu(x)
    v8, deq_v = pqk.quantize_e4m3(to_dev_bf16(x["v"]))
    o, lse = pqk.varlen_attn_fwd_fp8(q8, k8, v8, torch.cat([deq_qk, deq_v]).contiguous(), to_dev(x["cu_seqlens"]),
                                     softmax_scale=0.1, want_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), a[0].view(torch.int16)) and torch.equal(lse, a[1])


# ---------------------------------------------------------------- FP8 output of the Q/K prologue

def _prologue_fp32_error(x, w_, pos, eps, base, rows, inv):
    """Absolute bound on the kernel's fp32 error in y * inv for every element:
    y = a cos(phi) - b sin(phi) (or a sin + b cos) with a, b the pair's
    normalised, weighted values. The sum of D squares in fp32 is off by at
    most D * 2^-24 relative, the reciprocal square root by 2 ulp, so a and b
    carry at most 2^-17 relative error for D <= 128; the fp32 sine and cosine
    of the reduced angle (|phi| <= pi) are off by at most 2^-21.41 absolute
    (CUDA's stated bound for __sincosf there); a handful of fp32 roundings
    add 2^-20 of the result. So |error| <= inv * ((|a| + |b|) * 2^-17 + |y| * 2^-20)."""
    zero = np.zeros_like(pos)
    a = np.abs(oracle.qk_norm_rope(x, w_, zero, eps, base, rows=rows))  # phi = 0: the unrotated values
    T, H, D = a.shape
    pair = a.reshape(T, H, D // 2, 2)[..., ::-1].reshape(T, H, D)  # interleaved pairs (2j, 2j+1)
    y = np.abs(oracle.qk_norm_rope(x, w_, pos, eps, base, rows=rows))
    return inv * ((a + pair) * 2.0 ** -17 + y * 2.0 ** -20), y * inv


def _check_prologue_e4m3(x, w, rows=None, stride_pad=0, what=""):
    """Codes and scales of pqk_qk_norm_rope_e4m3 against the oracle. The
    scales are equal bit for bit (the same float arithmetic on both sides).
    The kernel rounds fp32 values and the oracle float64 ones, so a code may
    differ only where the oracle's value lies within the kernel's fp32 error
    bound (_prologue_fp32_error) of an e4m3 rounding boundary, and then it
    must be the other neighbour of that boundary."""
    torch = torch_cuda()
    T, H, D = x["q"].shape
    if stride_pad:
        buf = torch.zeros((T, 2 * H * D + stride_pad), dtype=torch.bfloat16, device="cuda")
        buf[:, :H * D] = to_dev_bf16(x["q"]).view(T, H * D)
        buf[:, H * D + stride_pad:] = to_dev_bf16(x["k"]).view(T, H * D)
        q, k = buf[:, :H * D].view(T, H, D), buf[:, H * D + stride_pad:].view(T, H, D)
    else:
        q, k = to_dev_bf16(x["q"]), to_dev_bf16(x["k"])
    q8, k8, deq = pqk.qk_norm_rope_e4m3(q, k, to_dev_bf16(x["w_q"]), to_dev_bf16(x["w_k"]), to_dev(x["pos"]),
                                         eps=w.eps, rope_base=w.rope_base)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    d = deq.cpu().numpy()
    sel = np.arange(T) if rows is None else rows
    ties = total = 0
    for i, (name, codes) in enumerate((("q", q8), ("k", k8))):
        rc, rdeq = oracle.qk_norm_rope_e4m3(x[name], x["w_" + name], x["pos"], w.eps, w.rope_base, rows=rows)
        assert np.all(d[i * H:(i + 1) * H] == rdeq), f"{what}: {name} scale"
        g = codes.cpu().numpy()[sel]
        mism = g != rc
        if mism.any():
            inv = 1.0 / float(rdeq)
            err, scaled = _prologue_fp32_error(x[name], x["w_" + name], x["pos"], w.eps, w.rope_base, rows, inv)
            y = oracle.qk_norm_rope(x[name], x["w_" + name], x["pos"], w.eps, w.rope_base, rows=rows)
            v = y[mism] * inv
            gv = _decode(g[mism])
            step = _e4m3_quantum(np.abs(v))
            bad = np.abs(gv - v) > step * 0.5 + err[mism]
            assert not bad.any(), (f"{what}: {name} code off by more than a rounding boundary plus the fp32 bound: "
                                   f"{gv[bad][:4]} vs {v[bad][:4]} (bound {err[mism][bad][:4]})")
        ties += int(mism.sum())
        total += g.size
    assert ties <= max(8, total // 200), f"{what}: {ties} of {total} codes differ"
    return q8, k8, deq


@pytest.mark.parametrize("cfg", [1, 2])
def test_prologue_e4m3_configs(cfg):
    w = wl.config(cfg)
    _check_prologue_e4m3(wl.prologue_inputs(w), w, what=f"configuration {cfg}")


@pytest.mark.parametrize("D", [64, 128])
def test_prologue_e4m3_ragged_and_strided(D):
    w = wl.custom([300, 0, 17, 129], H=6, D=D, seed=51)
    _check_prologue_e4m3(wl.prologue_inputs(w), w, stride_pad=64, what=f"ragged strided D{D}")


def test_prologue_e4m3_58048_tokens_sampled():
    w = wl.config(3)
    _check_prologue_e4m3(wl.prologue_inputs(w), w, rows=wl.sample_rows(w, 256), what="58,048 tokens")


def test_prologue_e4m3_feeds_the_fp8_attention():
    # the fused prologue's codes in the FP8 Q K^T attention = the plain
    # attention on their dequantised values
    torch = torch_cuda()
    w = wl.custom([700, 1300], H=4, D=128, seed=52)
    x = wl.prologue_inputs(w)
    v = wl.attention_inputs(w)["v"]
    q8, k8, deq = _check_prologue_e4m3(x, w, what="feeds the attention")
    scale = 1.0 / math.sqrt(128)
    o, lse = pqk.varlen_attn_fwd_fp8qk(q8, k8, to_dev_bf16(v), deq, to_dev(w.cu_seqlens()), softmax_scale=scale,
                                       want_lse=True)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    H = w.H
    dq = deq.cpu().numpy().astype(np.float64)
    qd = _decode(q8.cpu().numpy()) * dq[None, :H, None]
    kd = _decode(k8.cpu().numpy()) * dq[None, H:, None]
    ro, rl = oracle.varlen_attn(qd, kd, wl.bf16_bits_to_f64(v), w.cu_seqlens(), scale)
    assert_attention(bf16_to_f64(o), ro, "fused prologue -> FP8 attention")
    assert max_abs(lse.cpu().numpy().astype(np.float64).T, rl) <= LSE_MAX_ABS
