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
