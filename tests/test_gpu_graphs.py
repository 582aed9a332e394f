"""The block call under CUDA-graph capture: every entry point enqueues only
kernels and stream-ordered operations on the caller's stream (tensor maps
are encoded on the host and passed by value), so a serving loop can capture
qk_norm_rope -> varlen attention -> modulate_swiglu once and replay it.
Replays must reproduce the direct calls bit for bit. The first call on a
device sets up the library's per-device state, so it is made before the
capture, as the header asks."""

import numpy as np
import pytest

from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import to_dev, to_dev_bf16, torch_cuda

pytestmark = pytest.mark.gpu


def _block(torch, w, d, o):
    pqk.qk_norm_rope(d["q"], d["k"], d["w_q"], d["w_k"], d["pos"], eps=w.eps, rope_base=w.rope_base,
                     q_out=o["qn"], k_out=o["kn"])
    pqk.varlen_attn_fwd(o["qn"], o["kn"], d["v"], d["cu"], o=o["o"], workspace=o["ws"])
    pqk.modulate_swiglu(d["x"], d["shift"], d["scale"], d["cu"], gate_res=d["gate_res"],
                        branch=o["o"].view(w.T, w.C), gate=d["gate"], up=d["up"], eps=w.eps, x_out=o["x_out"],
                        h=o["h"], act=o["act"])


@pytest.mark.parametrize("lens, H, D", [([200, 312], 4, 64), ([1000, 0, 2000], 8, 128)])
def test_captured_block_call_replays_bitwise(lens, H, D):
    torch = torch_cuda()
    w = wl.custom(lens, H, D, seed=13)
    p, a, e = wl.prologue_inputs(w), wl.attention_inputs(w), wl.epilogue_inputs(w, with_branch=False)
    d = {"q": to_dev_bf16(p["q"]), "k": to_dev_bf16(p["k"]), "v": to_dev_bf16(a["v"]),
         "w_q": to_dev_bf16(p["w_q"]), "w_k": to_dev_bf16(p["w_k"]), "pos": to_dev(p["pos"]),
         "cu": to_dev(w.cu_seqlens()), "x": to_dev_bf16(e["x"]), "gate": to_dev_bf16(e["gate"]),
         "up": to_dev_bf16(e["up"]), "shift": to_dev(e["shift"]), "scale": to_dev(e["scale"]),
         "gate_res": to_dev(e["gate_res"])}
    o = {"qn": torch.empty_like(d["q"]), "kn": torch.empty_like(d["k"]), "o": torch.empty_like(d["q"]),
         "x_out": torch.empty_like(d["x"]), "h": torch.empty_like(d["x"]),
         "act": torch.empty((w.T, w.F), dtype=torch.bfloat16, device="cuda"),
         "ws": torch.empty(pqk.varlen_attn_workspace_size(w.B), dtype=torch.uint8, device="cuda")}
    _block(torch, w, d, o)                       # direct call (also the first call on the device)
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in o.items() if k != "ws"}
    for v in o.values():
        v.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            _block(torch, w, d, o)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    for k, v in ref.items():
        assert torch.equal(o[k].view(torch.int16) if o[k].dtype == torch.bfloat16 else o[k],
                           v.view(torch.int16) if v.dtype == torch.bfloat16 else v), k
    del g


def test_captured_linear_layers_replay_bitwise():
    """The fused-epilogue GEMMs (tensor maps encoded on the host, passed by
    value) captured once: the O-projection writing x', W1 with SwiGLU, and W2
    adding its gated branch to x'; replays equal the direct calls bit for
    bit."""
    torch = torch_cuda()
    w = wl.custom([300, 0, 700], 4, 64, C=256, F=384, seed=17)
    lo, l1, l2 = (wl.linear_inputs(w, n) for n in ("o_proj", "w1", "w2"))
    a, wo, w1, w2 = to_dev_bf16(lo["a"]), to_dev_bf16(lo["w"]), to_dev_bf16(l1["w"]), to_dev_bf16(l2["w"])
    x, gr, cu = to_dev_bf16(lo["x"]), to_dev(lo["gate_res"]), to_dev(lo["cu_seqlens"])
    h = to_dev_bf16(l1["a"])
    xp, act, x2 = torch.empty_like(x), torch.empty((w.T, w.F), dtype=torch.bfloat16, device="cuda"), torch.empty_like(x)

    def layers():
        pqk.linear_gated_residual(a, wo, x=x, gate_res=gr, cu_seqlens=cu, out=xp)
        pqk.linear_swiglu(h, w1, act=act)
        pqk.linear_gated_residual(act, w2, x=xp, gate_res=gr, cu_seqlens=cu, out=x2)

    layers()                                     # direct calls (the first on the device precede capture)
    torch.cuda.synchronize()
    ref = [t.clone() for t in (xp, act, x2)]
    for t in (xp, act, x2):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            layers()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    for got, want in zip((xp, act, x2), ref):
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    del g
