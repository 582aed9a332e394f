"""Writes tests/golden/oracle_tiny_config.json: oracle outputs on the tiny
packed-attention configuration (2 requests of 200 and 312 tokens, 4 heads,
head_dim 64, hidden 256, ffn 512, seed 0), for the three block operations
and for every widened variant (see variants()). Calls only the oracle and the
seeded input generators, so the stored numbers guard the oracle against
unintended drift; they carry no authority of their own beyond that.

Run from the repository root:  python tests/golden/make_golden.py
"""

import json
import math
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import oracle  # noqa: E402
from packed_attention_qk_b200 import workloads as wl  # noqa: E402

ROWS = [0, 1, 199, 200, 311, 511]


def summarise(a):
    a = np.asarray(a, np.float64)
    return {"sum": float(a.sum()), "abs_sum": float(np.abs(a).sum()), "sq_sum": float((a * a).sum())}


def variants(w, p, a):
    """The widened rows on the same configuration: three-axis RoPE (the
    200-token request laid out as a 2 x 10 x 10 grid, sections 8 / 12 / 12),
    the full-width norm, block skipping at tau = 4 on block-scaled inputs
    (blocks of 16 query rows x 64 keys, tiles of 64 rows), attention with FP8
    Q, K and with FP8 Q, K, V, P (the definition, the online schedule with
    blocks of 64 keys and threshold 4, and the definition with block skipping
    at tau = 4 on the block-scaled inputs), and the three linear layers with
    their fused epilogues."""
    out = {}
    scale = 1.0 / math.sqrt(w.D)
    y = oracle.qk_norm_rope_3axis(p["q"], p["w_q"], w.positions3(video_grid=(2, 10, 10)), (8, 12, 12), w.eps,
                                  w.rope_base)
    out["q_norm_rope_3axis"] = {"summary": summarise(y), "head0": [y[r, 0, :8].tolist() for r in ROWS]}
    y = oracle.qk_fullc_norm_rope(p["q"], wl.fullc_weights(w)["w_q"], p["pos"], w.eps, w.rope_base)
    out["q_fullc_norm_rope"] = {"summary": summarise(y), "head0": [y[r, 0, :8].tolist() for r in ROWS]}
    b = wl.block_scaled_attention_inputs(w)
    o, lse, counts = oracle.varlen_attn_skip(b["q"], b["k"], b["v"], b["cu_seqlens"], scale, 4.0, block=(16, 64),
                                             tile_rows=64)
    out["attn_skip_tau4"] = {"summary": summarise(o), "lse_summary": summarise(lse), "counts": list(counts),
                             "head0": [o[r, 0, :8].tolist() for r in ROWS]}
    o, lse, _, _, deq = oracle.varlen_attn_fp8qk(a["q"], a["k"], a["v"], a["cu_seqlens"], scale)
    out["attn_fp8qk"] = {"summary": summarise(o), "lse_summary": summarise(lse), "deq": deq.tolist(),
                         "head0": [o[r, 0, :8].tolist() for r in ROWS]}
    o, lse, deq = oracle.varlen_attn_fp8(a["q"], a["k"], a["v"], a["cu_seqlens"], scale)
    out["attn_fp8"] = {"summary": summarise(o), "lse_summary": summarise(lse), "deq": deq.tolist(),
                       "head0": [o[r, 0, :8].tolist() for r in ROWS]}
    o, lse, deq = oracle.varlen_attn_fp8_online(a["q"], a["k"], a["v"], a["cu_seqlens"], scale, kblock=64,
                                                threshold=4.0)
    out["attn_fp8_online_64_4"] = {"summary": summarise(o), "lse_summary": summarise(lse), "deq": deq.tolist(),
                                   "head0": [o[r, 0, :8].tolist() for r in ROWS]}
    counts = []
    o, lse, deq = oracle.varlen_attn_fp8(b["q"], b["k"], b["v"], b["cu_seqlens"], scale, tau=4.0, skip_block=(16, 64),
                                         skip_tile_rows=64, counts_out=counts)
    out["attn_fp8_skip_tau4"] = {"summary": summarise(o), "lse_summary": summarise(lse), "counts": list(counts[0]),
                                 "head0": [o[r, 0, :8].tolist() for r in ROWS]}
    for name in ("o_proj", "w1", "w2"):
        d = wl.linear_inputs(w, name)
        if name == "w1":
            y = oracle.linear_swiglu(d["a"], d["w"])
        else:
            y = oracle.linear_gated_residual(d["a"], d["w"], d["x"], d["gate_res"], d["cu_seqlens"])
        out[f"linear_{name}"] = {"summary": summarise(y), "first": [y[r, :8].tolist() for r in ROWS]}
    return out


def main():
    w = wl.config(1)
    p = wl.prologue_inputs(w)
    a = wl.attention_inputs(w)
    e = wl.epilogue_inputs(w, with_branch=True)
    out = {"config": w.name, "rows": ROWS, "values_per_row": 8}
    for style, tag in ((oracle.ROPE_INTERLEAVED, "interleaved"), (oracle.ROPE_HALF, "half")):
        y = oracle.qk_norm_rope(p["q"], p["w_q"], p["pos"], w.eps, w.rope_base, style)
        out[f"q_norm_rope_{tag}"] = {"summary": summarise(y), "head0": [y[r, 0, :8].tolist() for r in ROWS]}
    o, lse = oracle.varlen_attn(a["q"], a["k"], a["v"], a["cu_seqlens"], 1.0 / math.sqrt(w.D))
    out["attn_o"] = {"summary": summarise(o), "head0": [o[r, 0, :8].tolist() for r in ROWS]}
    out["attn_lse"] = {"summary": summarise(lse), "rows": [lse[r].tolist() for r in ROWS]}
    xo, h, act = oracle.modulate_swiglu(e["x"], e["shift"], e["scale"], e["gate_res"], e["cu_seqlens"],
                                        branch=e["branch"], gate=e["gate"], up=e["up"], eps=w.eps)
    for name, t in (("x_out", xo), ("h", h), ("act", act)):
        out[name] = {"summary": summarise(t), "first": [t[r, :8].tolist() for r in ROWS]}
    out.update(variants(w, p, a))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_config.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
