"""GPU parity of pqk_qk_norm_rope and pqk_modulate_swiglu against the
float64 oracle ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长", section
"融合 DiT 算子"; "MiniMax H3 FastH3 real-time serving with vLLM-Omni",
bullet "Fused DiT operators")."""

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import assert_elementwise, bf16_to_f64, to_dev, to_dev_bf16, torch_cuda

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- qk_norm_rope

def prologue_case(w, style, rows=None, in_place=True):
    torch = torch_cuda()
    x = wl.prologue_inputs(w)
    q, k = to_dev_bf16(x["q"]), to_dev_bf16(x["k"])
    wq, wk, pos = to_dev_bf16(x["w_q"]), to_dev_bf16(x["w_k"]), to_dev(x["pos"])
    if in_place:
        qo, ko = pqk.qk_norm_rope(q, k, wq, wk, pos, eps=w.eps, rope_base=w.rope_base, style=style)
    else:
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        pqk.qk_norm_rope(q, k, wq, wk, pos, eps=w.eps, rope_base=w.rope_base, style=style, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    for name, out, wname in (("q", qo, "w_q"), ("k", ko, "w_k")):
        ref = oracle.qk_norm_rope(x[name], x[wname], x["pos"], w.eps, w.rope_base, style, rows=rows)
        got = bf16_to_f64(out) if rows is None else bf16_to_f64(out[torch.from_numpy(rows).long().cuda()])
        assert_elementwise(got, ref, f"{w.name} {name} style {style}")


@pytest.mark.parametrize("style", [pqk.ROPE_INTERLEAVED, pqk.ROPE_HALF])
@pytest.mark.parametrize("cfg", [1, 2])
def test_qk_norm_rope_full(cfg, style):
    prologue_case(wl.config(cfg), style)


@pytest.mark.parametrize("style", [pqk.ROPE_INTERLEAVED, pqk.ROPE_HALF])
def test_qk_norm_rope_out_of_place_ragged(style):
    # odd head count (2H rows not a multiple of a warp step), T not a multiple of anything
    w = wl.custom([37, 0, 1, 129], H=5, D=128, seed=41)
    prologue_case(w, style, in_place=False)
    w = wl.custom([3, 250], H=3, D=64, seed=42)
    prologue_case(w, style, in_place=False)


@pytest.mark.parametrize("D", [64, 128])
def test_qk_norm_rope_into_wider_output_rows_with_guard_bands(D):
    # outputs with their own token strides: Q and K written into two slots of
    # a wider row (as into a sequence-parallel send buffer), inputs
    # contiguous; everything outside the two slots keeps its canary value
    torch = torch_cuda()
    w = wl.custom([300, 0, 17, 129], H=6, D=D, seed=43)
    x = wl.prologue_inputs(w)
    T, H = w.T, w.H
    q, k = to_dev_bf16(x["q"]), to_dev_bf16(x["k"])
    wq, wk, pos = to_dev_bf16(x["w_q"]), to_dev_bf16(x["w_k"]), to_dev(x["pos"])
    width = 3 * H * D + 64
    buf = torch.full((T + 2, width), 7.0, dtype=torch.bfloat16, device="cuda")
    qo = buf[1:1 + T, 32:32 + H * D].view(T, H, D)
    ko = buf[1:1 + T, 32 + H * D:32 + 2 * H * D].view(T, H, D)
    pqk.qk_norm_rope(q, k, wq, wk, pos, eps=w.eps, rope_base=w.rope_base, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    for name, out, wname in (("q", qo, "w_q"), ("k", ko, "w_k")):
        ref = oracle.qk_norm_rope(x[name], x[wname], x["pos"], w.eps, w.rope_base)
        assert_elementwise(bf16_to_f64(out), ref, f"{name} into a wider row")
    guard = torch.cat([buf[0], buf[T + 1], buf[1:1 + T, :32].flatten(), buf[1:1 + T, 32 + 2 * H * D:].flatten()])
    assert bool((guard == 7.0).all())


def test_qk_norm_rope_58048_tokens_sampled():
    w = wl.config(3)
    prologue_case(w, pqk.ROPE_INTERLEAVED, rows=wl.sample_rows(w, 512))


@pytest.mark.parametrize("T", wl.C5_TOKENS)
def test_qk_norm_rope_sweep_40_heads_sampled(T):
    w = wl.config(5, T)
    prologue_case(w, pqk.ROPE_INTERLEAVED, rows=wl.sample_rows(w, 512))


def test_qk_norm_rope_fused_qkv_rows():
    torch = torch_cuda()
    w = wl.custom([100, 60], H=4, D=128, seed=43)
    x = wl.prologue_inputs(w)
    T, H, D = w.T, w.H, w.D
    qkv = torch.zeros((T, 3 * H * D), dtype=torch.bfloat16, device="cuda")
    qkv[:, :H * D] = to_dev_bf16(x["q"]).view(T, H * D)
    qkv[:, H * D:2 * H * D] = to_dev_bf16(x["k"]).view(T, H * D)
    v_before = qkv[:, 2 * H * D:].clone()
    q = qkv[:, :H * D].view(T, H, D)
    k = qkv[:, H * D:2 * H * D].view(T, H, D)
    pqk.qk_norm_rope(q, k, to_dev_bf16(x["w_q"]), to_dev_bf16(x["w_k"]), to_dev(x["pos"]), eps=w.eps)
    torch.cuda.synchronize()
    assert torch.equal(qkv[:, 2 * H * D:], v_before)
    assert_elementwise(bf16_to_f64(q), oracle.qk_norm_rope(x["q"], x["w_q"], x["pos"], w.eps, w.rope_base), "q")
    assert_elementwise(bf16_to_f64(k), oracle.qk_norm_rope(x["k"], x["w_k"], x["pos"], w.eps, w.rope_base), "k")


def test_qk_norm_rope_deterministic():
    torch = torch_cuda()
    w = wl.config(2)
    x = wl.prologue_inputs(w)
    outs = []
    for _ in range(3):
        q, k = to_dev_bf16(x["q"]), to_dev_bf16(x["k"])
        pqk.qk_norm_rope(q, k, to_dev_bf16(x["w_q"]), to_dev_bf16(x["w_k"]), to_dev(x["pos"]))
        outs.append((q, k))
    torch.cuda.synchronize()
    for q, k in outs[1:]:
        assert torch.equal(q.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(k.view(torch.int16), outs[0][1].view(torch.int16))


# ---------------------------------------------------------------- three-axis RoPE

SECTIONS = {128: (16, 24, 24), 64: (8, 12, 12)}


def prologue3_case(w, style, grid, rows=None):
    torch = torch_cuda()
    x = wl.prologue_inputs(w)
    pos3 = w.positions3(grid)
    q, k = to_dev_bf16(x["q"]), to_dev_bf16(x["k"])
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    sec = SECTIONS[w.D]
    pqk.qk_norm_rope_3axis(q, k, to_dev_bf16(x["w_q"]), to_dev_bf16(x["w_k"]), to_dev(pos3), sec, eps=w.eps,
                           rope_base=w.rope_base, style=style, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.from_numpy(rows).long().cuda()])
    for name, out, wname in (("q", qo, "w_q"), ("k", ko, "w_k")):
        ref = oracle.qk_norm_rope_3axis(x[name], x[wname], pos3, sec, w.eps, w.rope_base, style, rows=rows)
        assert_elementwise(bf16_to_f64(sel(out)), ref, f"{w.name} {name} three-axis style {style}")


@pytest.mark.parametrize("style", [pqk.ROPE_INTERLEAVED, pqk.ROPE_HALF])
def test_qk_norm_rope_3axis_small_video_grids(style):
    # a joint sequence whose video run is a 3 x 5 x 7 latent grid (D 128), and
    # a D 64 one with a 2 x 4 x 6 grid
    w = wl.Workload("text 9 + audio 4 + video 3x5x7", 60, [9 + 4 + 105], H=3, D=128, C=384, F=64,
                    pos_runs=[[9, 4, 105]])
    prologue3_case(w, style, (3, 5, 7))
    w = wl.Workload("text 5 + video 2x4x6", 61, [5 + 48], H=2, D=64, C=128, F=64, pos_runs=[[5, 48]])
    prologue3_case(w, style, (2, 4, 6))


def test_qk_norm_rope_3axis_58048_tokens_sampled():
    w = wl.config(3)
    prologue3_case(w, pqk.ROPE_INTERLEAVED, (12, 48, 96), rows=wl.sample_rows(w, 1024))


def test_qk_norm_rope_3axis_with_equal_ids_is_bitwise_the_one_axis_kernel():
    torch = torch_cuda()
    w = wl.config(2)
    x = wl.prologue_inputs(w)
    pos = x["pos"]
    pos3 = np.ascontiguousarray(np.stack([pos, pos, pos], 1))
    a = [to_dev_bf16(x["q"]), to_dev_bf16(x["k"])]
    b = [to_dev_bf16(x["q"]), to_dev_bf16(x["k"])]
    wq, wk = to_dev_bf16(x["w_q"]), to_dev_bf16(x["w_k"])
    pqk.qk_norm_rope(a[0], a[1], wq, wk, to_dev(pos))
    pqk.qk_norm_rope_3axis(b[0], b[1], wq, wk, to_dev(pos3), SECTIONS[w.D])
    torch.cuda.synchronize()
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))


# ---------------------------------------------------------------- full-width Q/K norm

def fullc_case(w, style, rows=None):
    torch = torch_cuda()
    x = wl.prologue_inputs(w)
    fw = wl.fullc_weights(w)
    q, k = to_dev_bf16(x["q"]), to_dev_bf16(x["k"])
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    pqk.qk_fullc_norm_rope(q, k, to_dev_bf16(fw["w_q"]), to_dev_bf16(fw["w_k"]), to_dev(x["pos"]), eps=w.eps,
                           rope_base=w.rope_base, style=style, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.from_numpy(rows).long().cuda()])
    for name, out, wname in (("q", qo, "w_q"), ("k", ko, "w_k")):
        ref = oracle.qk_fullc_norm_rope(x[name], fw[wname], x["pos"], w.eps, w.rope_base, style, rows=rows)
        assert_elementwise(bf16_to_f64(sel(out)), ref, f"{w.name} {name} full width style {style}")


@pytest.mark.parametrize("style", [pqk.ROPE_INTERLEAVED, pqk.ROPE_HALF])
def test_qk_fullc_norm_rope_small(style):
    fullc_case(wl.config(1), style)
    fullc_case(wl.custom([37, 0, 90], H=5, D=128, seed=62), style)
    fullc_case(wl.custom([50], H=3, D=64, seed=63), style)


def test_qk_fullc_norm_rope_58048_tokens_sampled():
    w = wl.config(3)
    fullc_case(w, pqk.ROPE_INTERLEAVED, rows=wl.sample_rows(w, 512))


def test_qk_fullc_norm_rope_one_head_is_bitwise_the_per_head_kernel():
    torch = torch_cuda()
    w = wl.custom([300], H=1, D=128, seed=64)
    x = wl.prologue_inputs(w)
    a = [to_dev_bf16(x["q"]), to_dev_bf16(x["k"])]
    b = [to_dev_bf16(x["q"]), to_dev_bf16(x["k"])]
    wq, wk, pos = to_dev_bf16(x["w_q"]), to_dev_bf16(x["w_k"]), to_dev(x["pos"])
    pqk.qk_norm_rope(a[0], a[1], wq, wk, pos)
    pqk.qk_fullc_norm_rope(b[0], b[1], wq, wk, pos)
    torch.cuda.synchronize()
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))


# ---------------------------------------------------------------- modulate_swiglu

def epilogue_case(w, norm_type=pqk.NORM_RMS, with_branch=False, rows=None, fused_gate_up=False, swiglu=True):
    torch = torch_cuda()
    e = wl.epilogue_inputs(w, with_branch=with_branch)
    x = to_dev_bf16(e["x"])
    shift, scale, gres = to_dev(e["shift"]), to_dev(e["scale"]), to_dev(e["gate_res"])
    cu = to_dev(e["cu_seqlens"])
    br = to_dev_bf16(e["branch"]) if with_branch else None
    gate = up = None
    if swiglu:
        if fused_gate_up:
            gu = torch.empty((w.T, 2 * w.F), dtype=torch.bfloat16, device="cuda")
            gu[:, :w.F] = to_dev_bf16(e["gate"])
            gu[:, w.F:] = to_dev_bf16(e["up"])
            gate, up = gu[:, :w.F], gu[:, w.F:]
        else:
            gate, up = to_dev_bf16(e["gate"]), to_dev_bf16(e["up"])
    x_out = torch.empty_like(x) if with_branch else None
    xo, h, act = pqk.modulate_swiglu(x, shift, scale, cu, gate_res=gres, branch=br, gate=gate, up=up,
                                     norm_type=norm_type, eps=w.eps, x_out=x_out)
    torch.cuda.synchronize()
    rxo, rh, ract = oracle.modulate_swiglu(e["x"], e["shift"], e["scale"], e["gate_res"], e["cu_seqlens"],
                                           norm_type=norm_type, eps=w.eps, branch=e.get("branch"),
                                           gate=e["gate"] if swiglu else None, up=e["up"] if swiglu else None,
                                           rows=rows)
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.from_numpy(rows).long().cuda()])
    assert_elementwise(bf16_to_f64(sel(h)), rh, f"{w.name} h")
    if with_branch:
        assert_elementwise(bf16_to_f64(sel(xo)), rxo, f"{w.name} x_out")
    if swiglu:
        assert_elementwise(bf16_to_f64(sel(act)), ract, f"{w.name} act")


@pytest.mark.parametrize("with_branch", [False, True])
@pytest.mark.parametrize("norm_type", [pqk.NORM_RMS, pqk.NORM_LAYER, pqk.NORM_NONE])
def test_modulate_swiglu_tiny_config(norm_type, with_branch):
    epilogue_case(wl.config(1), norm_type=norm_type, with_branch=with_branch)


@pytest.mark.parametrize("with_branch", [False, True])
def test_modulate_swiglu_4096_tokens(with_branch):
    epilogue_case(wl.config(2), with_branch=with_branch, fused_gate_up=True)


def test_modulate_swiglu_ragged_requests_and_widths():
    # several requests incl. empty ones, C not a multiple of the block width
    w = wl.custom([5, 0, 130, 1, 0, 64], H=3, D=40, C=120, F=72, seed=51)
    epilogue_case(w, with_branch=True)
    epilogue_case(w, norm_type=pqk.NORM_LAYER, with_branch=True, swiglu=False)
    w = wl.custom([77], H=1, D=8, C=16384, F=8, seed=52)
    epilogue_case(w, with_branch=True)


def test_modulate_swiglu_four_requests_sampled():
    w = wl.config(4)
    epilogue_case(w, with_branch=True, rows=wl.sample_rows(w, 128))


@pytest.mark.parametrize("T", wl.C5_TOKENS)
def test_modulate_swiglu_sweep_sampled(T):
    w = wl.config(5, T)
    epilogue_case(w, rows=wl.sample_rows(w, 512))


def test_modulate_swiglu_in_place_outputs():
    torch = torch_cuda()
    w = wl.custom([90, 38], H=2, D=64, seed=53)
    e = wl.epilogue_inputs(w, with_branch=True)
    x = to_dev_bf16(e["x"])
    gu = torch.empty((w.T, 2 * w.F), dtype=torch.bfloat16, device="cuda")
    gu[:, :w.F] = to_dev_bf16(e["gate"])
    gu[:, w.F:] = to_dev_bf16(e["up"])
    gate, up = gu[:, :w.F], gu[:, w.F:]
    # x' back into x, h into a separate buffer, act into a contiguous copy of
    # gate; h must come from x' (formed once from the original x), for both
    # norms that read the row more than once
    for norm_type in (pqk.NORM_RMS, pqk.NORM_LAYER):
        x = to_dev_bf16(e["x"])
        act = gate.contiguous()
        _, h, _ = pqk.modulate_swiglu(x, to_dev(e["shift"]), to_dev(e["scale"]), to_dev(e["cu_seqlens"]),
                                      gate_res=to_dev(e["gate_res"]), branch=to_dev_bf16(e["branch"]), gate=act,
                                      up=up.contiguous(), x_out=x, act=act, norm_type=norm_type)
        torch.cuda.synchronize()
        rxo, rh, ract = oracle.modulate_swiglu(e["x"], e["shift"], e["scale"], e["gate_res"], e["cu_seqlens"],
                                               branch=e["branch"], gate=e["gate"], up=e["up"], norm_type=norm_type)
        assert_elementwise(bf16_to_f64(x), rxo, "x in place")
        assert_elementwise(bf16_to_f64(h), rh, "h with x' written over x")
        assert_elementwise(bf16_to_f64(act), ract, "act in place")
