"""The oracle still reproduces its stored outputs on the tiny configuration
(tests/golden/oracle_tiny_config.json, written by tests/golden/make_golden.py
from the oracle alone). A change to the oracle's arithmetic that moves these
numbers must say which passage of the pages, or which reading of it,
justifies it."""

import json
import math
import os

import numpy as np

from oracle import oracle
from packed_attention_qk_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_config.json")


def _summary_close(a, s):
    a = np.asarray(a, np.float64)
    for key, val in (("sum", a.sum()), ("abs_sum", np.abs(a).sum()), ("sq_sum", (a * a).sum())):
        assert abs(val - s[key]) <= 1e-9 * max(1.0, abs(s[key])), key


def test_oracle_matches_stored_tiny_config_outputs():
    g = json.load(open(GOLDEN))
    rows = g["rows"]
    w = wl.config(1)
    p = wl.prologue_inputs(w)
    for style, tag in ((oracle.ROPE_INTERLEAVED, "interleaved"), (oracle.ROPE_HALF, "half")):
        y = oracle.qk_norm_rope(p["q"], p["w_q"], p["pos"], w.eps, w.rope_base, style)
        _summary_close(y, g[f"q_norm_rope_{tag}"]["summary"])
        np.testing.assert_allclose([y[r, 0, :8] for r in rows], g[f"q_norm_rope_{tag}"]["head0"], atol=1e-12)
    a = wl.attention_inputs(w)
    o, lse = oracle.varlen_attn(a["q"], a["k"], a["v"], a["cu_seqlens"], 1.0 / math.sqrt(w.D))
    _summary_close(o, g["attn_o"]["summary"])
    _summary_close(lse, g["attn_lse"]["summary"])
    np.testing.assert_allclose([o[r, 0, :8] for r in rows], g["attn_o"]["head0"], atol=1e-12)
    np.testing.assert_allclose([lse[r] for r in rows], g["attn_lse"]["rows"], atol=1e-12)
    e = wl.epilogue_inputs(w, with_branch=True)
    xo, h, act = oracle.modulate_swiglu(e["x"], e["shift"], e["scale"], e["gate_res"], e["cu_seqlens"],
                                        branch=e["branch"], gate=e["gate"], up=e["up"], eps=w.eps)
    for name, t in (("x_out", xo), ("h", h), ("act", act)):
        _summary_close(t, g[name]["summary"])
        np.testing.assert_allclose([t[r, :8] for r in rows], g[name]["first"], atol=1e-12)


def test_oracle_variants_match_stored_tiny_config_outputs():
    g = json.load(open(GOLDEN))
    rows = g["rows"]
    w = wl.config(1)
    p, a = wl.prologue_inputs(w), wl.attention_inputs(w)
    scale = 1.0 / math.sqrt(w.D)
    y = oracle.qk_norm_rope_3axis(p["q"], p["w_q"], w.positions3(video_grid=(2, 10, 10)), (8, 12, 12), w.eps,
                                  w.rope_base)
    _summary_close(y, g["q_norm_rope_3axis"]["summary"])
    np.testing.assert_allclose([y[r, 0, :8] for r in rows], g["q_norm_rope_3axis"]["head0"], atol=1e-12)
    y = oracle.qk_fullc_norm_rope(p["q"], wl.fullc_weights(w)["w_q"], p["pos"], w.eps, w.rope_base)
    _summary_close(y, g["q_fullc_norm_rope"]["summary"])
    np.testing.assert_allclose([y[r, 0, :8] for r in rows], g["q_fullc_norm_rope"]["head0"], atol=1e-12)
    b = wl.block_scaled_attention_inputs(w)
    o, lse, counts = oracle.varlen_attn_skip(b["q"], b["k"], b["v"], b["cu_seqlens"], scale, 4.0, block=(16, 64),
                                             tile_rows=64)
    assert list(counts) == g["attn_skip_tau4"]["counts"]
    _summary_close(o, g["attn_skip_tau4"]["summary"])
    _summary_close(lse, g["attn_skip_tau4"]["lse_summary"])
    np.testing.assert_allclose([o[r, 0, :8] for r in rows], g["attn_skip_tau4"]["head0"], atol=1e-12)
    online = lambda *x: oracle.varlen_attn_fp8_online(*x, kblock=64, threshold=4.0)
    for key, fn in (("attn_fp8qk", oracle.varlen_attn_fp8qk), ("attn_fp8", oracle.varlen_attn_fp8),
                    ("attn_fp8_online_64_4", online)):
        res = fn(a["q"], a["k"], a["v"], a["cu_seqlens"], scale)
        o, lse, deq = res[0], res[1], res[-1]
        assert np.array_equal(np.asarray(deq, np.float32), np.asarray(g[key]["deq"], np.float32))
        _summary_close(o, g[key]["summary"])
        _summary_close(lse, g[key]["lse_summary"])
        np.testing.assert_allclose([o[r, 0, :8] for r in rows], g[key]["head0"], atol=1e-12)
    counts = []
    o, lse, _ = oracle.varlen_attn_fp8(b["q"], b["k"], b["v"], b["cu_seqlens"], scale, tau=4.0, skip_block=(16, 64),
                                       skip_tile_rows=64, counts_out=counts)
    assert list(counts[0]) == g["attn_fp8_skip_tau4"]["counts"]
    _summary_close(o, g["attn_fp8_skip_tau4"]["summary"])
    _summary_close(lse, g["attn_fp8_skip_tau4"]["lse_summary"])
    np.testing.assert_allclose([o[r, 0, :8] for r in rows], g["attn_fp8_skip_tau4"]["head0"], atol=1e-12)
    for name in ("o_proj", "w1", "w2"):
        d = wl.linear_inputs(w, name)
        if name == "w1":
            y = oracle.linear_swiglu(d["a"], d["w"])
        else:
            y = oracle.linear_gated_residual(d["a"], d["w"], d["x"], d["gate_res"], d["cu_seqlens"])
        _summary_close(y, g[f"linear_{name}"]["summary"])
        np.testing.assert_allclose([y[r, :8] for r in rows], g[f"linear_{name}"]["first"], atol=1e-12)
