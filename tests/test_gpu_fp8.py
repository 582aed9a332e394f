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
from tests.gpu_utils import (LSE_MAX_ABS, assert_attention, bf16_to_f64, max_abs, rel_l2, to_dev, to_dev_bf16,
                             torch_cuda)

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

def _full_fp8_gpu(x, scale):
    torch = torch_cuda()
    q8, k8, deq_qk = _quantise_gpu(x)
    v8, deq_v = pqk.quantize_e4m3(to_dev_bf16(x["v"]))
    deq = torch.cat([deq_qk, deq_v]).contiguous()
    o, lse = pqk.varlen_attn_fwd_fp8(q8, k8, v8, deq, to_dev(x["cu_seqlens"]), softmax_scale=scale, want_lse=True)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    return o, lse, v8, deq


def _check_full_fp8(x, scale, what, rows=None):
    """Element-wise against the oracle, each row allowed, beyond the attention
    tolerance, one e4m3 step (2^-4 relative) of its largest-weight key: the
    kernel rounds fp32 probabilities, the oracle float64 ones, so a value
    lying on an e4m3 rounding boundary may round differently."""
    o, lse, v8, deq = _full_fp8_gpu(x, scale)
    ro, rl, rdeq = oracle.varlen_attn_fp8(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, rows=rows)
    T, H, D = x["q"].shape
    assert np.array_equal(deq.cpu().numpy(), rdeq)
    sel = np.arange(T) if rows is None else rows
    g = bf16_to_f64(o)[sel]
    assert rel_l2(g, ro) <= 1e-2, what
    # largest softmax weight per (row, head), from the dequantised Q, K
    q8, k8, _ = _quantise_gpu(x)
    dq = deq.cpu().numpy().astype(np.float64)
    import torch
    dec = lambda c: torch.from_numpy(c.cpu().numpy()).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    qd, kd = dec(q8) * dq[None, :H, None], dec(k8) * dq[None, H:2 * H, None]
    vmax = float(np.abs(dec(v8)).max() * dq[2 * H:].max())
    cu = x["cu_seqlens"]
    for n, t in enumerate(sel):
        i = int(np.searchsorted(cu, t, side="right") - 1)
        lo, hi = int(cu[i]), int(cu[i + 1])
        for h in range(H):
            s = scale * (kd[lo:hi, h] @ qd[t, h])
            wmax = float(np.exp(s - s.max()).max() / np.exp(s - s.max()).sum())
            err = float(np.max(np.abs(g[n, h] - ro[n, h])))
            assert err <= 2e-2 + 2.0 ** -3 * wmax * vmax, f"{what}: row {t} head {h} error {err:.3e}"
    assert max_abs(lse.cpu().numpy().astype(np.float64).T[sel], rl) <= LSE_MAX_ABS


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
    _check_full_fp8(x, 1.0 / math.sqrt(128), "full fp8 peaked")


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
    for o, lse, _, _ in a[1:]:
        assert torch.equal(o.view(torch.int16), a[0][0].view(torch.int16)) and torch.equal(lse, a[0][1])
