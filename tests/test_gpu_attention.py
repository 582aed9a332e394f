"""GPU parity of pqk_varlen_attn_fwd against the float64 oracle.

Packed requests, bidirectional inside each request and nothing across, only
valid tokens processed ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长",
section "长序列注意力与通信优化"). Small cases are compared element by element
on every output; the full-size configurations on a seeded sample of query
rows (first and last row of every request included).
"""

import math

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import (LSE_MAX_ABS, assert_attention, bf16_to_f64, max_abs, to_dev, to_dev_bf16,
                             torch_cuda)

pytestmark = pytest.mark.gpu


def run_gpu(x, H, D, want_lse=True, scale=None):
    torch = torch_cuda()
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    cu = to_dev(x["cu_seqlens"])
    o, lse = pqk.varlen_attn_fwd(q, k, v, cu, softmax_scale=scale, want_lse=want_lse)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    return bf16_to_f64(o), (lse.cpu().numpy().astype(np.float64) if want_lse else None)


def check(x, H, D, rows=None, what="", peaked=False, scale=None):
    scale = scale if scale is not None else 1.0 / math.sqrt(D)
    o, lse = run_gpu(x, H, D, scale=scale)
    ro, rl = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, rows=rows)
    sel = slice(None) if rows is None else rows
    assert_attention(o[sel], ro, what, peaked=peaked)
    assert max_abs(lse.T[sel], rl) <= LSE_MAX_ABS, f"{what}: lse max-abs {max_abs(lse.T[sel], rl):.3e}"


def custom_inputs(lens, H, D, seed, q_scale=1.0):
    w = wl.custom(lens, H, D, seed=seed)
    x = wl.attention_inputs(w)
    if q_scale != 1.0:
        q = wl.bf16_bits_to_f32(x["q"]) * np.float32(q_scale)
        x["q"] = wl.f32_to_bf16_bits(q)
    return w, x


def test_tiny_config_full():
    w = wl.config(1)
    check(wl.attention_inputs(w), w.H, w.D, what="2 requests 200+312, H4 D64")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("lens", [[1], [127], [128], [129], [255, 256, 257], [300, 0, 513, 1],
                                  [0, 0, 700], [384, 17, 2, 640]])
def test_ragged_lengths_full(lens, D):
    w, x = custom_inputs(lens, 3, D, seed=sum(lens) + D)
    check(x, w.H, w.D, what=f"lens {lens} D{D}")


def test_many_requests():
    g = np.random.default_rng(11)
    lens = [int(v) for v in g.integers(0, 400, 60)]
    w, x = custom_inputs(lens, 2, 128, seed=12)
    check(x, w.H, w.D, what="60 requests")


@pytest.mark.parametrize("n_req", [3000, 9000])
def test_thousands_of_short_requests(n_req):
    # above 8,192 requests the schedule keeps the given order instead of
    # longest first; both must give every row its own request's attention
    g = np.random.default_rng(n_req)
    lens = [int(v) for v in g.integers(0, 40, n_req)]
    lens[n_req // 2] = 300
    w, x = custom_inputs(lens, 2, 64, seed=n_req)
    rows = np.sort(g.choice(w.T, size=512, replace=False)).astype(np.int32)
    check(x, w.H, w.D, rows=rows, what=f"{n_req} requests")


@pytest.mark.parametrize("D", [64, 128])
def test_peaked_scores(D):
    # Q x 8: the softmax concentrates on a few keys, O is close to single V rows
    w, x = custom_inputs([200, 700], 2, D, seed=21, q_scale=8.0)
    check(x, w.H, w.D, what="peaked", peaked=True)


def test_non_default_scale():
    w, x = custom_inputs([333, 129], 2, 128, seed=22)
    check(x, w.H, w.D, what="scale 0.3", scale=0.3)


def test_joint_sequence_4096_sampled():
    w = wl.config(2)
    x = wl.attention_inputs(w)
    check(x, w.H, w.D, rows=wl.sample_rows(w, 256), what="4096 tokens H16")


def test_joint_sequence_58048_sampled():
    w = wl.config(3)
    x = wl.attention_inputs(w)
    check(x, w.H, w.D, rows=wl.sample_rows(w, 256), what="58,048 tokens H24")


@pytest.mark.parametrize("outliers", [False, True])
def test_four_request_batch_sampled(outliers):
    w = wl.config(4)
    x = wl.attention_inputs(w, outliers=outliers)
    check(x, w.H, w.D, rows=wl.sample_rows(w, 64), what=f"4 requests outliers={outliers}")


def _tail_rows(w, per_segment):
    """Seeded sample rows plus, in every request, the rows of its last
    (ragged) 128-row tile and the first rows after each 256-row boundary of
    the last two tiles."""
    rows = set(int(r) for r in wl.sample_rows(w, per_segment))
    cu = w.cu_seqlens()
    for i in range(len(cu) - 1):
        lo, hi = int(cu[i]), int(cu[i + 1])
        if hi == lo:
            continue
        last = lo + ((hi - lo - 1) // 128) * 128
        rows.update(range(last, hi, 7))
        rows.update((hi - 1, hi - 2, max(lo, last - 1)))
    return np.array(sorted(rows), np.int32)


@pytest.mark.parametrize("config", [3, 4])
def test_peaked_full_size_sampled_with_ragged_tails(config):
    # Q x 8 at the full-size configurations: O is close to single V rows, so
    # the unit-scale bound applies; the sample covers every request's ragged
    # last tile
    w = wl.config(config)
    x = wl.attention_inputs(w)
    x["q"] = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(x["q"]) * np.float32(8.0))
    check(x, w.H, w.D, rows=_tail_rows(w, 32), what=f"peaked Q x 8, configuration {config}", peaked=True)


def test_strided_fused_qkv_and_output_canaries():
    torch = torch_cuda()
    lens = [300, 45]
    T, H, D = sum(lens), 2, 128
    w, x = custom_inputs(lens, H, D, seed=31)
    qkv = torch.empty((T, 3, H, D), dtype=torch.bfloat16, device="cuda")
    for i, n in enumerate(("q", "k", "v")):
        qkv[:, i] = to_dev_bf16(x[n])
    # output rows with a guard band of 8 rows on each side and a wider row
    o_full = torch.full((T + 16, H * D + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    o = o_full[8:8 + T, :H * D].view(T, H, D)
    pqk.varlen_attn_fwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], to_dev(x["cu_seqlens"]), o=o)
    torch.cuda.synchronize()
    ro, _ = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], 1.0 / math.sqrt(D))
    assert_attention(bf16_to_f64(o), ro, "strided")
    guard = torch.cat([o_full[:8].flatten(), o_full[8 + T:].flatten(), o_full[8:8 + T, H * D:].flatten()])
    assert bool((guard == 7.0).all())


def test_deterministic_bitwise():
    torch = torch_cuda()
    w = wl.config(2)
    x = wl.attention_inputs(w)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    cu = to_dev(x["cu_seqlens"])
    outs = []
    for _ in range(3):
        o, lse = pqk.varlen_attn_fwd(q, k, v, cu, want_lse=True)
        outs.append((o.clone(), lse.clone()))
    torch.cuda.synchronize()
    for o, lse in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(lse, outs[0][1])


@pytest.mark.parametrize("cu", [[0, 100, 50, 200], [0, 100, 150], [1, 100, 200]])
def test_bad_cu_seqlens_sets_status_and_writes_nothing(cu):
    torch = torch_cuda()
    T, H, D = 200, 2, 64
    q = torch.randn((T, H, D), device="cuda").to(torch.bfloat16)
    o = torch.full_like(q, 3.0)
    pqk.varlen_attn_fwd(q, q, q, torch.tensor(cu, dtype=torch.int32, device="cuda"), o=o)
    assert pqk.get_device_status() == -7
    assert bool((o == 3.0).all())
    assert pqk.get_device_status() == 0   # read-and-clear
