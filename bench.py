"""Benchmark of one DiT-block hot-path step on B200.

A step is one block call over one request of the 58,048-token joint
text + audio + video sequence (24 heads x 128, hidden 3,072, FFN 8,192):
  qk_norm_rope (Q, K)  ->  varlen_attn_fwd (Q, K, V)  ->
  modulate_swiglu (x + gate_res * O as the gated residual, adaLN
  modulation, SwiGLU on gate / up),
all through the C ABI of libpqk. The dense projections between them are
outside the hot path; seeded synthetic tensors stand in for their outputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). ``value`` is attention FLOPs of all ranks
per second of device time of the whole step (max over ranks); the kernel
figures and the roofline of the dominant kernel (the attention) are in the
same line. With N > 1 (torchrun) every rank runs its own request: weak
scaling, no collective on the data path.

After the timed steps the same line also carries, under ``kernels``: the
three-axis RoPE, back-to-back and full-width norm timings; the block-
skipping attention on the local-attention stand-in (``--skip-tau``, plain
vs skipping vs FP8 Q K^T and the whole attention in FP8, each with and
without skipping); the FP8 Q K^T attention
on the step's inputs, and the Q/K prologue with e4m3 output against the
prologue followed by the separate quantisation (``--no-fp8`` leaves them out); the block's three linear
layers with the gated residual or SwiGLU in the GEMM epilogue, on the step's
own activations, against cuBLAS plus torch epilogues (``linear_epilogue``;
``--no-linear`` leaves it out); the two HBM-bound kernels on the 40-head
bandwidth-sweep shapes at 4,096 and 58,048 tokens with an L2 flush between
launches (``bandwidth_sweep_40_heads``; ``--no-bw-sweep`` leaves it out); and,
with ``--graph``,
the step replayed as a CUDA graph (``graph_ms_per_step``). ``--config N``
selects another configuration, ``--sweep`` the HBM bandwidth sweep,
``--linear-sweep`` the fused-epilogue linear layers on a range of shapes.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "varlen attn TFLOP/s @58k tokens (% bf16 peak); fused DiT-op HBM GB/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_traffic.json")
ATTN_SRC = os.path.join(ROOT, "packed_attention_qk_b200", "csrc", "varlen_attn_fwd.cu")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=3, help="workload number (3 = 58,048-token joint sequence)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="one request of this many tokens with the shape of --config (a smaller case for profiling)")
    ap.add_argument("--sweep", action="store_true",
                    help="prologue/epilogue bandwidth sweep (40 heads x 128; hidden 5,120, FFN 13,824) instead "
                         "of the step; one JSON line per kernel and token count")
    ap.add_argument("--outliers", action="store_true",
                    help="K with 0.1%% of its entries scaled x20 (the outlier variant of the 4-request batch)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="leave out the FP8 Q K^T attention timing")
    ap.add_argument("--linear-sweep", action="store_true",
                    help="the fused-epilogue linear layers alone against cuBLAS on a range of token counts and "
                         "widths (one JSON line per shape) instead of the step")
    ap.add_argument("--no-linear", action="store_true",
                    help="leave out the linear layers with the fused epilogues (gated residual, SwiGLU)")
    ap.add_argument("--no-bw-sweep", action="store_true",
                    help="leave out the HBM-bound kernels on the 40-head sweep shapes at 4,096 and 58,048 tokens")
    ap.add_argument("--no-pairs", action="store_true",
                    help="leave out the step's attention timed again on CTA pairs (pqk_set_attn_cta_pairs)")
    ap.add_argument("--graph", action="store_true",
                    help="also time the block call captured once in a CUDA graph and replayed (graph_ms_per_step)")
    ap.add_argument("--skip-tau", type=float, default=8.0,
                    help="threshold (log2 units) of the block-skipping attention timed on the local-attention "
                         "stand-in after the steps; negative = leave that timing out")
    return ap.parse_args()


def peaks():
    try:
        d = json.load(open(PEAKS_FILE))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def attn_traffic():
    """Per-launch DRAM bytes of the attention kernel from a committed ncu
    capture, or None when the kernel source changed since."""
    try:
        d = json.load(open(TRAFFIC_FILE))
    except Exception:
        return None
    if d.get("source_sha256_16") != source_hash(ATTN_SRC):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, enabled=True):
        self.gpu, self.enabled, self.lines, self.proc = gpu_index, enabled, [], None

    def __enter__(self):
        if self.enabled:
            try:
                self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                              "-i", str(self.gpu), "-lms", "200"], stdout=subprocess.PIPE,
                                             stderr=subprocess.DEVNULL, text=True)
                self.t = threading.Thread(target=self._read, daemon=True)
                self.t.start()
            except Exception:
                self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ inputs

def make_inputs(w, device, outliers=False):
    import torch
    from packed_attention_qk_b200 import workloads as wl

    def dev16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    p = wl.prologue_inputs(w)
    if outliers:
        p["k"] = wl.bf16_k_with_outliers(w.seed, (w.T, w.H, w.D))
    a = {"v": wl.bf16_normal(w.seed, "v", (w.T, w.H, w.D))}
    e = wl.epilogue_inputs(w, with_branch=False)
    d = {"q": dev16(p["q"]), "k": dev16(p["k"]), "v": dev16(a["v"]), "w_q": dev16(p["w_q"]),
         "w_k": dev16(p["w_k"]), "pos": torch.from_numpy(p["pos"]).to(device),
         "cu": torch.from_numpy(w.cu_seqlens()).to(device), "x": dev16(e["x"]), "gate": dev16(e["gate"]),
         "up": dev16(e["up"]), "shift": torch.from_numpy(e["shift"]).to(device),
         "scale": torch.from_numpy(e["scale"]).to(device), "gate_res": torch.from_numpy(e["gate_res"]).to(device)}
    return d


def alloc_outputs(w, d):
    import torch
    from packed_attention_qk_b200 import pqk
    o = {"qn": torch.empty_like(d["q"]), "kn": torch.empty_like(d["k"]), "o": torch.empty_like(d["q"]),
         "x_out": torch.empty_like(d["x"]), "h": torch.empty_like(d["x"]),
         "act": torch.empty((w.T, w.F), dtype=torch.bfloat16, device=d["x"].device),
         "ws": torch.empty(pqk.varlen_attn_workspace_size(w.B), dtype=torch.uint8, device=d["x"].device)}
    return o


def block_call(w, d, o, ev=None):
    """One step: the three C-ABI calls on the current stream. ``ev`` (4
    events) brackets the kernels for per-kernel device times."""
    from packed_attention_qk_b200 import pqk
    if ev:
        ev[0].record()
    pqk.qk_norm_rope(d["q"], d["k"], d["w_q"], d["w_k"], d["pos"], eps=w.eps, rope_base=w.rope_base,
                     q_out=o["qn"], k_out=o["kn"])
    if ev:
        ev[1].record()
    pqk.varlen_attn_fwd(o["qn"], o["kn"], d["v"], d["cu"], o=o["o"], workspace=o["ws"])
    if ev:
        ev[2].record()
    pqk.modulate_swiglu(d["x"], d["shift"], d["scale"], d["cu"], gate_res=d["gate_res"],
                        branch=o["o"].view(w.T, w.C), gate=d["gate"], up=d["up"], eps=w.eps, x_out=o["x_out"],
                        h=o["h"], act=o["act"])
    if ev:
        ev[3].record()


LAUNCHES_PER_STEP = 4  # qk_norm_rope, schedule builder, attention, modulate_swiglu


def time_linear_layers(w, d, o, pk, pk_kind, reps=3):
    """The block's three linear layers with their fused epilogues on the
    step's own activations (attention output, h, act) and random-init
    weights: the output projection and W2 with the gated residual, W1 with
    SwiGLU. Each is timed against cuBLAS (torch's linear) followed by the
    same epilogue as torch element-wise kernels, and the GEMM alone (ours
    without epilogue vs cuBLAS)."""
    import torch
    import torch.nn.functional as Fnn
    from packed_attention_qk_b200 import pqk
    from packed_attention_qk_b200 import workloads as wl
    dev = d["x"].device

    def dev_w(name, n_out, n_in):
        bits = wl.bf16_linear_weight(w.seed, name, n_out, n_in)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    T, Cd, F = w.T, w.C, w.F
    w_o, w1, w2 = dev_w("w_o", Cd, Cd), dev_w("w1", 2 * F, Cd), dev_w("w2", Cd, F)
    a_o = o["o"].view(T, w.H * w.D)
    x, gr, cu = d["x"], d["gate_res"], d["cu"]
    # torch's epilogue broadcasts one gate row (one request) or gathers one per token
    gr_tok = gr[0] if w.B == 1 else torch.repeat_interleave(gr, torch.tensor(w.seg_lens, device=dev), dim=0)
    out_c, out_f = torch.empty_like(x), torch.empty_like(o["act"])
    layers = {
        "o_proj": (lambda: pqk.linear_gated_residual(a_o, w_o, x=x, gate_res=gr, cu_seqlens=cu, out=out_c),
                   lambda: pqk.linear_gated_residual(a_o, w_o, out=out_c),
                   lambda: Fnn.linear(a_o, w_o),
                   lambda: torch.addcmul(x, gr_tok, Fnn.linear(a_o, w_o)),
                   2.0 * T * (w.H * w.D) * Cd),
        "w1_swiglu": (lambda: pqk.linear_swiglu(o["h"], w1, act=out_f),
                      None,
                      lambda: Fnn.linear(o["h"], w1),
                      lambda: (lambda y: Fnn.silu(y[:, :F]) * y[:, F:])(Fnn.linear(o["h"], w1)),
                      2.0 * T * Cd * 2 * F),
        "w2": (lambda: pqk.linear_gated_residual(o["act"], w2, x=x, gate_res=gr, cu_seqlens=cu, out=out_c),
               lambda: pqk.linear_gated_residual(o["act"], w2, out=out_c),
               lambda: Fnn.linear(o["act"], w2),
               lambda: torch.addcmul(x, gr_tok, Fnn.linear(o["act"], w2)),
               2.0 * T * F * Cd),
    }
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def ms(fn):
        fn()
        torch.cuda.synchronize()
        ev[0].record()
        for _ in range(reps):
            fn()
        ev[1].record()
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1]) / reps

    res, fused_total, unfused_total, flops_total = {}, 0.0, 0.0, 0.0
    for name, (fused, gemm_only, cublas, cublas_epi, flops) in layers.items():
        f_ms = ms(fused)
        r = {"fused_ms": f_ms, "fused_tflops": flops / (f_ms * 1e-3) / 1e12,
             "cublas_gemm_ms": ms(cublas), "cublas_plus_torch_epilogue_ms": ms(cublas_epi)}
        if gemm_only is not None:
            r["gemm_only_ms"] = ms(gemm_only)
        r["speedup_vs_cublas_plus_epilogue"] = r["cublas_plus_torch_epilogue_ms"] / f_ms
        res[name] = r
        fused_total += f_ms
        unfused_total += r["cublas_plus_torch_epilogue_ms"]
        flops_total += flops
    if pqk.get_device_status() != 0:
        raise RuntimeError("device status set during the linear-layer timing")
    tflops = flops_total / (fused_total * 1e-3) / 1e12
    res.update({"fused_total_ms": fused_total, "unfused_total_ms": unfused_total,
                "speedup_vs_cublas_plus_epilogue": unfused_total / fused_total, "fused_tflops": tflops,
                "frac_of_bf16_burst": tflops / pk["bf16_tflops"], "peak_kind": f"{pk_kind} bf16 burst",
                "weights": "random-init N(0, 1/in) bf16"})
    del w_o, w1, w2, out_c, out_f
    return res


def time_bandwidth_sweep(w_step, dev, pk, pk_kind, tokens=(4096, 58048), reps=10):
    """The two HBM-bound kernels on the 40-head bandwidth-sweep shapes (Q, K
    [T, 40, 128]; modulation + SwiGLU with hidden 5,120 and FFN 13,824, no
    residual branch) at the given token counts: one launch at a time, a
    256 MB write between launches to flush L2 (the 4,096-token working set is
    close to its 126 MB), followed by a 256 MB read that evicts the written
    lines (their write-back would otherwise compete with the kernel), median
    of ``reps`` launches after two warm-up ones.
    Inputs are drawn on the device with the sweep's distributions (torch's
    CUDA generator, seeded per token count) to keep the multi-GB tensors off
    the host; the kernels' time does not depend on the values."""
    import torch
    from packed_attention_qk_b200 import pqk
    from packed_attention_qk_b200 import workloads as wl
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clean = torch.ones(64 << 20, dtype=torch.int32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def timed(fn):
        ts = []
        for i in range(2 + reps):
            # write 256 MB (more than the L2), then read another 256 MB so that
            # the written lines are evicted before the kernel starts rather
            # than written back while it runs
            flush.fill_(i & 0xFF)
            clean.sum()
            ev[0].record()
            fn()
            ev[1].record()
            torch.cuda.synchronize()
            if i >= 2:
                ts.append(ev[0].elapsed_time(ev[1]))
        return statistics.median(ts)

    out = {}
    for T in tokens:
        w = wl.config(5, T)
        gen = torch.Generator(device=dev)
        gen.manual_seed(w.seed * 1000003 + T)
        bf = lambda *shape: torch.randn(*shape, generator=gen, device=dev).to(torch.bfloat16)
        q, k = bf(T, w.H, w.D), bf(T, w.H, w.D)
        wq = (torch.rand(w.D, generator=gen, device=dev) + 0.5).to(torch.bfloat16)
        wk = (torch.rand(w.D, generator=gen, device=dev) + 0.5).to(torch.bfloat16)
        pos = torch.arange(T, dtype=torch.int32, device=dev)
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        pro_ms = timed(lambda: pqk.qk_norm_rope(q, k, wq, wk, pos, eps=w.eps, rope_base=w.rope_base, q_out=qo,
                                                k_out=ko))
        del q, k, qo, ko
        x = bf(T, w.C)
        gate, up = bf(T, w.F), bf(T, w.F)
        shift = torch.randn(1, w.C, generator=gen, device=dev) * 0.1
        scale = torch.randn(1, w.C, generator=gen, device=dev) * 0.1
        cu = torch.tensor([0, T], dtype=torch.int32, device=dev)
        h, act = torch.empty_like(x), torch.empty_like(gate)
        epi_ms = timed(lambda: pqk.modulate_swiglu(x, shift, scale, cu, gate=gate, up=up, eps=w.eps, h=h, act=act))
        del x, gate, up, h, act
        if pqk.get_device_status() != 0:
            raise RuntimeError("device status set during the bandwidth sweep")
        pro_gbs = w.prologue_bytes() / (pro_ms * 1e-3) / 1e9
        epi_gbs = w.epilogue_bytes() / (epi_ms * 1e-3) / 1e9
        out[str(T)] = {"qk_norm_rope_us": pro_ms * 1e3, "qk_norm_rope_gbs": pro_gbs,
                       "qk_norm_rope_frac_hbm": pro_gbs / pk["hbm_gbs"],
                       "modulate_swiglu_us": epi_ms * 1e3, "modulate_swiglu_gbs": epi_gbs,
                       "modulate_swiglu_frac_hbm": epi_gbs / pk["hbm_gbs"]}
    del flush, clean
    torch.cuda.empty_cache()
    out["shapes"] = "qk_norm_rope: Q, K [T, 40, 128]; modulate_swiglu: hidden 5,120, FFN 13,824, no branch"
    out["peak"] = f"{pk_kind} HBM {pk['hbm_gbs']:.1f} GB/s"
    out["l2"] = "between launches 256 MB written, then another 256 MB read (the L2 holds no dirty lines at the start)"
    return out


# ------------------------------------------------------------------ CPU oracle

def cpu_baseline_sample(w, rows_per_request, seed_rows=None, threads=None):
    """Times the oracle's attention on a seeded sample of query rows (all
    heads, full keys), on `threads` OpenMP threads (all of them by default).
    Returns (TFLOP/s, seconds, rows, threads)."""
    from oracle import oracle
    from packed_attention_qk_b200 import workloads as wl
    x = wl.attention_inputs(w)
    rows = wl.sample_rows(w, rows_per_request)
    if threads is not None:
        all_threads = oracle.num_threads()
        oracle.set_num_threads(threads)
        try:
            return cpu_baseline_sample(w, rows_per_request, seed_rows)
        finally:
            oracle.set_num_threads(all_threads)
    cu = w.cu_seqlens()
    seg = np.searchsorted(cu, rows, side="right") - 1
    flops = float(sum(4.0 * w.H * w.D * (cu[s + 1] - cu[s]) for s in seg))
    t0 = time.perf_counter()
    oracle.varlen_attn(x["q"], x["k"], x["v"], cu, 1.0 / math.sqrt(w.D), rows=rows)
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, dt, int(len(rows)), oracle.num_threads()


def cpu_elementwise_sample(w, n_tokens=16384):
    """Times the oracle's Q/K norm + RoPE and its modulation + SwiGLU on a
    seeded sample of the step's tokens (the step's shapes, residual branch
    on). Returns ({qk_norm_rope_gbs, modulate_swiglu_gbs}, seconds, tokens)."""
    from oracle import oracle
    from packed_attention_qk_b200 import workloads as wl
    p = wl.prologue_inputs(w)
    e = wl.epilogue_inputs(w, with_branch=True)
    rows = np.sort(np.random.default_rng(w.seed + 2000).choice(w.T, size=min(n_tokens, w.T), replace=False))
    rows = rows.astype(np.int32)
    t0 = time.perf_counter()
    oracle.qk_norm_rope(p["q"], p["w_q"], p["pos"], w.eps, w.rope_base, rows=rows)
    oracle.qk_norm_rope(p["k"], p["w_k"], p["pos"], w.eps, w.rope_base, rows=rows)
    t1 = time.perf_counter()
    oracle.modulate_swiglu(e["x"], e["shift"], e["scale"], e["gate_res"], e["cu_seqlens"], eps=w.eps,
                           branch=e["branch"], gate=e["gate"], up=e["up"], rows=rows)
    t2 = time.perf_counter()
    n = len(rows)
    pro = w.prologue_bytes() / w.T * n / (t1 - t0) / 1e9
    epi = w.epilogue_bytes(with_branch=True) / w.T * n / (t2 - t1) / 1e9
    return {"qk_norm_rope_gbs": pro, "modulate_swiglu_gbs": epi}, t2 - t0, n


# ------------------------------------------------------------------ arms

def run_reference(args, w):
    """The oracle, as it stands, on host cores: each step is the attention
    over a bounded seeded sample of query rows of the same workload."""
    from oracle import oracle
    from packed_attention_qk_b200 import workloads as wl
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = wl.attention_inputs(w)
    cu = w.cu_seqlens()
    rows = wl.sample_rows(w, 16)
    seg = np.searchsorted(cu, rows, side="right") - 1
    flops = float(sum(4.0 * w.H * w.D * (cu[s + 1] - cu[s]) for s in seg))
    for _ in range(args.warmup):
        oracle.varlen_attn(x["q"], x["k"], x["v"], cu, 1.0 / math.sqrt(w.D), rows=rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.varlen_attn(x["q"], x["k"], x["v"], cu, 1.0 / math.sqrt(w.D), rows=rows)
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    sample = f"{len(rows)} query rows x {w.H} heads x all {w.T} keys per step (float64 oracle)"
    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": w.name, "tokens": w.T, "heads": w.H, "head_dim": w.D},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


class Ranks:
    """Process-group plumbing of a multi-rank run: a barrier and the maximum
    of a value over ranks (the device time of the slowest rank). With one
    rank both are no-ops. The same calls in the same order on every rank."""

    def __init__(self, world: int, device):
        self.world, self.device = world, device

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float) -> float:
        if self.world == 1:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())


def throughput(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def run_ours(args, w):
    import torch
    import torch.distributed as dist
    from packed_attention_qk_b200 import pqk

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    ranks = Ranks(world, dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max

    d = make_inputs(w, dev, outliers=args.outliers)
    o = alloc_outputs(w, d)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        block_call(w, d, o)
    torch.cuda.synchronize()
    if pqk.get_device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, enabled=not args.no_clocks) as clocks:
        barrier()
        torch.cuda.synchronize()
        start.record()
        for i in range(K):
            block_call(w, d, o, evs[i])
        stop.record()
        torch.cuda.synchronize()
        barrier()
    total_ms = max_over_ranks(start.elapsed_time(stop))
    if pqk.get_device_status() != 0:
        raise RuntimeError("device status set during the timed steps")
    graph_ms = None
    if args.graph:
        # the same block call captured once (all calls were made before, so
        # the library's per-device setup is done) and replayed K times
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs):
            with torch.cuda.graph(g, stream=cs):
                block_call(w, d, o)
        torch.cuda.current_stream().wait_stream(cs)
        for _ in range(args.warmup):
            g.replay()
        barrier()
        torch.cuda.synchronize()
        gs, gt = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        gs.record()
        for _ in range(K):
            g.replay()
        gt.record()
        torch.cuda.synchronize()
        barrier()
        graph_ms = max_over_ranks(gs.elapsed_time(gt)) / K
        if pqk.get_device_status() != 0:
            raise RuntimeError("device status set during the graph replays")
        del g
    pro = [e[0].elapsed_time(e[1]) for e in evs]
    att = [e[1].elapsed_time(e[2]) for e in evs]
    epi = [e[2].elapsed_time(e[3]) for e in evs]
    ms_step = total_ms / K
    flops = w.attn_flops()
    value = throughput(flops, world, ms_step)
    att_ms = statistics.mean(att)
    pk, pk_kind = peaks()
    attn_tflops = flops / (att_ms * 1e-3) / 1e12
    pro_gbs = w.prologue_bytes() / (statistics.mean(pro) * 1e-3) / 1e9
    epi_bytes = w.epilogue_bytes(with_branch=True)
    epi_gbs = epi_bytes / (statistics.mean(epi) * 1e-3) / 1e9

    # the three-axis RoPE variant on the same Q, K: (t, h, w) ids for the video
    # latent grid, one-axis ids repeated for text and audio
    pos3 = torch.from_numpy(w.positions3()).to(dev)
    sections = (w.D // 8, 3 * w.D // 16, 3 * w.D // 16)
    ev3 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for _ in range(2):
        pqk.qk_norm_rope_3axis(d["q"], d["k"], d["w_q"], d["w_k"], pos3, sections, eps=w.eps,
                               rope_base=w.rope_base, q_out=o["qn"], k_out=o["kn"])
    ev3[0].record()
    reps3 = 10
    for _ in range(reps3):
        pqk.qk_norm_rope_3axis(d["q"], d["k"], d["w_q"], d["w_k"], pos3, sections, eps=w.eps,
                               rope_base=w.rope_base, q_out=o["qn"], k_out=o["kn"])
    ev3[1].record()
    torch.cuda.synchronize()
    rope3_us = ev3[0].elapsed_time(ev3[1]) / reps3 * 1e3
    rope3_gbs = w.prologue_bytes(three_axis=True) / (rope3_us * 1e-6) / 1e9
    # the one-axis kernel timed the same way (back to back), for comparison
    ev3[0].record()
    for _ in range(reps3):
        pqk.qk_norm_rope(d["q"], d["k"], d["w_q"], d["w_k"], d["pos"], eps=w.eps, rope_base=w.rope_base,
                         q_out=o["qn"], k_out=o["kn"])
    ev3[1].record()
    torch.cuda.synchronize()
    rope1_b2b_us = ev3[0].elapsed_time(ev3[1]) / reps3 * 1e3
    # the full-width Q/K norm variant (weights of H*D entries), same way
    from packed_attention_qk_b200 import workloads as wl
    fw = wl.fullc_weights(w)
    fwq = torch.from_numpy(fw["w_q"].view(np.int16)).view(torch.bfloat16).to(dev)
    fwk = torch.from_numpy(fw["w_k"].view(np.int16)).view(torch.bfloat16).to(dev)
    pqk.qk_fullc_norm_rope(d["q"], d["k"], fwq, fwk, d["pos"], eps=w.eps, rope_base=w.rope_base, q_out=o["qn"],
                           k_out=o["kn"])
    ev3[0].record()
    for _ in range(reps3):
        pqk.qk_fullc_norm_rope(d["q"], d["k"], fwq, fwk, d["pos"], eps=w.eps, rope_base=w.rope_base,
                               q_out=o["qn"], k_out=o["kn"])
    ev3[1].record()
    torch.cuda.synchronize()
    fullc_us = ev3[0].elapsed_time(ev3[1]) / reps3 * 1e3
    fullc_gbs = (w.prologue_bytes() + 2 * w.H * w.D * 2) / (fullc_us * 1e-6) / 1e9

    # the step's attention on CTA pairs against the default one-SM kernel,
    # alternated, ten launches each, with the SM clock sampled meanwhile
    pairs = None
    if not args.no_pairs and w.D == 128:
        po = torch.empty_like(o["o"])
        run_attn = lambda: pqk.varlen_attn_fwd(o["qn"], o["kn"], d["v"], d["cu"], o=po, workspace=o["ws"])
        pt = {"one_sm": [], "pairs": []}
        pclk = {"one_sm": [], "pairs": []}
        try:
            for rnd in range(2):
                for name, on in (("one_sm", False), ("pairs", True)):
                    pqk.set_attn_cta_pairs(on)
                    run_attn()
                    torch.cuda.synchronize()
                    with ClockSampler(local, enabled=not args.no_clocks) as cs:
                        ev3[0].record()
                        for _ in range(10):
                            run_attn()
                        ev3[1].record()
                        torch.cuda.synchronize()
                    pt[name].append(ev3[0].elapsed_time(ev3[1]) / 10)
                    summ = cs.summary()
                    if summ and summ.get("sm_mhz"):
                        pclk[name].append(summ["sm_mhz"])
        finally:
            pqk.set_attn_cta_pairs(False)
        if pqk.get_device_status() != 0:
            raise RuntimeError("device status set during the CTA-pair timing")
        one_ms, pair_ms = min(pt["one_sm"]), min(pt["pairs"])
        pairs = {"one_sm_ms": one_ms, "pairs_ms": pair_ms, "pairs_tflops": flops / (pair_ms * 1e-3) / 1e12,
                 "speedup": one_ms / pair_ms,
                 "one_sm_sm_mhz": statistics.median(pclk["one_sm"]) if pclk["one_sm"] else None,
                 "pairs_sm_mhz": statistics.median(pclk["pairs"]) if pclk["pairs"] else None}
        del po

    # block skipping (Skip-Softmax) on the local-attention stand-in: Q and K
    # from sinusoids of the (t, h, w) ids plus noise, so that attention weight
    # sits on nearby tokens as in video; plain and skipping kernels on the
    # same inputs, and the share of dropped block decisions
    skip = None
    if args.skip_tau >= 0:
        lx = wl.local_attention_inputs(w, amplitude=16.0)
        lq, lk, lv = (torch.from_numpy(lx[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
        counts = torch.zeros(2, dtype=torch.int64, device=dev)
        lo = torch.empty_like(lq)
        plain = lambda: pqk.varlen_attn_fwd(lq, lk, lv, d["cu"], o=lo, workspace=o["ws"])
        skipping = lambda c=None: pqk.varlen_attn_fwd_skip(lq, lk, lv, d["cu"], args.skip_tau, o=lo,
                                                           workspace=o["ws"], skip_counts=c)
        plain()
        skipping(counts)
        torch.cuda.synchronize()
        times = {}
        for name, fn in (("plain", plain), ("skip", skipping), ("plain2", plain), ("skip2", skipping)):
            ev3[0].record()
            for _ in range(3):
                fn()
            ev3[1].record()
            torch.cuda.synchronize()
            times[name] = ev3[0].elapsed_time(ev3[1]) / 3
        if pqk.get_device_status() != 0:
            raise RuntimeError("device status set during the block-skipping timing")
        # the same with Q K^T in FP8 (SAGE reading), without and with skipping
        fp8_times = {}
        if w.D == 128:
            q8, k8, deq = pqk.quantize_qk_e4m3(lq, lk)
            fp8_plain = lambda: pqk.varlen_attn_fwd_fp8qk(q8, k8, lv, deq, d["cu"], o=lo, workspace=o["ws"])
            fp8_skip = lambda: pqk.varlen_attn_fwd_fp8qk(q8, k8, lv, deq, d["cu"], o=lo, workspace=o["ws"],
                                                         skip_threshold_log2=args.skip_tau)
            fp8_plain()
            fp8_skip()
            torch.cuda.synchronize()
            # the whole computation in FP8 (V and P too), without and with skipping
            lv8, ldeq_v = pqk.quantize_e4m3(lv)
            ldeq3 = torch.cat([deq, ldeq_v]).contiguous()
            full_plain = lambda: pqk.varlen_attn_fwd_fp8(q8, k8, lv8, ldeq3, d["cu"], o=lo, workspace=o["ws"])
            full_skip = lambda: pqk.varlen_attn_fwd_fp8(q8, k8, lv8, ldeq3, d["cu"], o=lo, workspace=o["ws"],
                                                        skip_threshold_log2=args.skip_tau)
            fp8_plain()
            fp8_skip()
            full_plain()
            full_skip()
            torch.cuda.synchronize()
            for name, fn in (("fp8", fp8_plain), ("fp8_skip", fp8_skip), ("full", full_plain),
                             ("full_skip", full_skip), ("fp8_2", fp8_plain), ("fp8_skip_2", fp8_skip),
                             ("full_2", full_plain), ("full_skip_2", full_skip)):
                ev3[0].record()
                for _ in range(3):
                    fn()
                ev3[1].record()
                torch.cuda.synchronize()
                fp8_times[name] = ev3[0].elapsed_time(ev3[1]) / 3
            if pqk.get_device_status() != 0:
                raise RuntimeError("device status set during the FP8 block-skipping timing")
            del q8, k8, lv8
        c = counts.cpu().tolist()
        n32 = sum(((L + 31) // 32) * ((L + 127) // 128) for L in w.seg_lens) * w.H
        n128 = sum(((L + 127) // 128) ** 2 for L in w.seg_lens) * w.H
        plain_ms = min(times["plain"], times["plain2"])
        skip_ms = min(times["skip"], times["skip2"])
        skip = {"input": "local-attention stand-in: Q, K = 16 x unit sinusoid features of the (t, h, w) ids "
                         "+ N(0, 1) noise, V ~ N(0, 1)",
                "tau_log2": args.skip_tau, "plain_ms": plain_ms, "skip_ms": skip_ms,
                "speedup": plain_ms / skip_ms, "dropped_block_share": c[0] / n32,
                "skipped_pv_share": c[1] / n128}
        if fp8_times:
            f_ms = min(fp8_times["fp8"], fp8_times["fp8_2"])
            fs_ms = min(fp8_times["fp8_skip"], fp8_times["fp8_skip_2"])
            ff_ms = min(fp8_times["full"], fp8_times["full_2"])
            ffs_ms = min(fp8_times["full_skip"], fp8_times["full_skip_2"])
            skip.update({"fp8qk_ms": f_ms, "fp8qk_skip_ms": fs_ms, "speedup_fp8qk_skip_vs_plain": plain_ms / fs_ms,
                         "full_fp8_ms": ff_ms, "full_fp8_skip_ms": ffs_ms,
                         "speedup_full_fp8_skip_vs_plain": plain_ms / ffs_ms})
        del lq, lk, lv, lo, lx

    # FP8 Q K^T (the SAGE reading): the step's normalised Q, K quantised per
    # head to e4m3, then the attention with S = Q K^T on the FP8 tensor cores
    fp8 = None
    if not args.no_fp8 and w.D == 128:
        q8, k8, deq = pqk.quantize_qk_e4m3(o["qn"], o["kn"])
        fo = torch.empty_like(o["o"])
        fp8_attn = lambda: pqk.varlen_attn_fwd_fp8qk(q8, k8, d["v"], deq, d["cu"], o=fo, workspace=o["ws"])
        fp8_attn()
        torch.cuda.synchronize()
        ev3[0].record()
        for _ in range(reps3):
            pqk.quantize_qk_e4m3(o["qn"], o["kn"], q8=q8, k8=k8, scales=None)
        ev3[1].record()
        torch.cuda.synchronize()
        quant_us = ev3[0].elapsed_time(ev3[1]) / reps3 * 1e3
        ev3[0].record()
        for _ in range(3):
            fp8_attn()
        ev3[1].record()
        torch.cuda.synchronize()
        fp8_ms = ev3[0].elapsed_time(ev3[1]) / 3
        if pqk.get_device_status() != 0:
            raise RuntimeError("device status set during the FP8 timing")
        # the whole computation in FP8: V quantised as well, P rounded to e4m3
        v8, deq_v = pqk.quantize_e4m3(d["v"])
        deq3 = torch.cat([deq, deq_v]).contiguous()
        full = lambda: pqk.varlen_attn_fwd_fp8(q8, k8, v8, deq3, d["cu"], o=fo, workspace=o["ws"])
        full()
        torch.cuda.synchronize()
        ev3[0].record()
        for _ in range(3):
            full()
        ev3[1].record()
        torch.cuda.synchronize()
        full_ms = ev3[0].elapsed_time(ev3[1]) / 3
        if pqk.get_device_status() != 0:
            raise RuntimeError("device status set during the FP8 timing")
        # the Q/K prologue with e4m3 output (the quantisation folded in, bound
        # scale): replaces qk_norm_rope + the separate quantisation pass
        pqk.qk_norm_rope_e4m3(d["q"], d["k"], d["w_q"], d["w_k"], d["pos"], eps=w.eps, rope_base=w.rope_base,
                              q8=q8, k8=k8)
        ev3[0].record()
        for _ in range(reps3):
            pqk.qk_norm_rope_e4m3(d["q"], d["k"], d["w_q"], d["w_k"], d["pos"], eps=w.eps, rope_base=w.rope_base,
                                  q8=q8, k8=k8)
        ev3[1].record()
        torch.cuda.synchronize()
        fused_us = ev3[0].elapsed_time(ev3[1]) / reps3 * 1e3
        fused_bytes = w.T * (6 * w.H * w.D + 4)
        fp8 = {"quantize_us": quant_us, "attn_ms": fp8_ms, "attn_tflops": flops / (fp8_ms * 1e-3) / 1e12,
               "prologue_e4m3_us": fused_us, "prologue_e4m3_gbs": fused_bytes / (fused_us * 1e-6) / 1e9,
               "prologue_e4m3_frac_hbm": fused_bytes / (fused_us * 1e-6) / 1e9 / pk["hbm_gbs"],
               "separate_prologue_and_quantize_us": rope1_b2b_us + quant_us,
               "speedup_vs_bf16": att_ms / fp8_ms,
               "quantize_gbs": (4 * w.T * w.H * w.D + 2 * w.T * w.H * w.D) / (quant_us * 1e-6) / 1e9,
               "full_fp8_attn_ms": full_ms, "full_fp8_speedup_vs_bf16": att_ms / full_ms}
        del q8, k8, v8, fo

    lin = None
    if not args.no_linear and w.H * w.D == w.C:
        lin = time_linear_layers(w, d, o, pk, pk_kind)

    # the HBM half of the metric on the bandwidth-sweep shapes (40 heads)
    bw = None if args.no_bw_sweep else time_bandwidth_sweep(w, dev, pk, pk_kind)

    # e2e through host buffers: every step copies all of its inputs from
    # pinned host memory to the device (H2D stream), runs the three C-ABI
    # calls (compute stream) and copies its outputs x', h, act back to pinned
    # host memory (D2H stream), all inside the timed region. Two device buffer
    # sets let step i+1's uploads and step i-1's downloads overlap step i's
    # kernels, as a serving loop would; events order each buffer set's reuse.
    e2e = None
    if not args.no_e2e:
        in_keys = ("q", "k", "v", "x", "gate", "up", "w_q", "w_k", "pos", "cu", "shift", "scale", "gate_res")
        out_keys = ("x_out", "h", "act")
        host_in = {k: d[k].cpu().pin_memory() for k in in_keys}
        host_out = [{k: torch.empty(o[k].shape, dtype=o[k].dtype, pin_memory=True) for k in out_keys}
                    for _ in range(2)]
        sets = [(d, o), ({k: torch.empty_like(d[k]) for k in in_keys}, alloc_outputs(w, d))]
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        e2e_steps = max(4, min(K, 8))

        def run_e2e(n):
            ev_in = [None, None]     # inputs of set b uploaded
            ev_done = [None, None]   # kernels of set b finished
            ev_out = [None, None]    # outputs of set b downloaded
            for i in range(n):
                b = i % 2
                dd, oo = sets[b]
                with torch.cuda.stream(s_in):
                    if ev_done[b] is not None:
                        s_in.wait_event(ev_done[b])      # set b's previous kernels have read their inputs
                    for k in in_keys:
                        dd[k].copy_(host_in[k], non_blocking=True)
                    ev_in[b] = torch.cuda.Event()
                    ev_in[b].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[b])
                    if ev_out[b] is not None:
                        s_cmp.wait_event(ev_out[b])      # set b's previous outputs are on the host
                    block_call(w, dd, oo)
                    ev_done[b] = torch.cuda.Event()
                    ev_done[b].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[b])
                    for k in out_keys:
                        host_out[b][k].copy_(oo[k], non_blocking=True)
                    ev_out[b] = torch.cuda.Event()
                    ev_out[b].record(s_out)

        run_e2e(2)
        torch.cuda.synchronize()
        barrier()
        s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(torch.cuda.current_stream())
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(torch.cuda.current_stream())
        run_e2e(e2e_steps)
        for st in (s_in, s_cmp, s_out):
            torch.cuda.current_stream().wait_stream(st)
        t2.record(torch.cuda.current_stream())
        torch.cuda.synchronize()
        barrier()
        if pqk.get_device_status() != 0:
            raise RuntimeError("device status set during the end-to-end steps")
        e2e_ms = max_over_ranks(s2.elapsed_time(t2)) / e2e_steps
        e2e = {"value": throughput(flops, world, e2e_ms), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
               "overlap": "two buffer sets: uploads and downloads overlap neighbouring steps' kernels"}
        del sets

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, secs, nrows, cores = cpu_baseline_sample(w, 96)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"attention of {nrows} seeded query rows x {w.H} heads over all keys of their request "
                         f"(float64 oracle, {secs:.1f} s)",
               "per_row_ms": secs / nrows * 1e3,
               "extrapolated_full_call_s": w.attn_flops() / (tf * 1e12),
               "extrapolation": "the whole attention at the sample's rate (not measured)"}
        tf1, secs1, nrows1, _ = cpu_baseline_sample(w, 4, threads=1)
        cpu["single_thread"] = {"value": tf1, "unit": "TFLOP/s", "cores": 1,
                                "sample": f"attention of {nrows1} seeded query rows x {w.H} heads "
                                          f"(float64 oracle, {secs1:.1f} s)"}
        el, el_secs, el_n = cpu_elementwise_sample(w)
        cpu["elementwise"] = {**el, "unit": "GB/s", "kind": "oracle",
                              "sample": f"Q/K norm + RoPE and modulation + SwiGLU (residual branch on) of {el_n} "
                                        f"seeded tokens of the step, counted as their algorithmic bytes "
                                        f"(float64 oracle, {el_secs:.1f} s)"}

    traffic = attn_traffic()
    peak = pk["bf16_tflops_sustained"]
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name + (" (K outliers)" if args.outliers else ""), "tokens_per_gpu": w.T,
                   "requests_per_gpu": w.B, "heads": w.H,
                   "head_dim": w.D, "hidden": w.C, "ffn": w.F,
                   "l2": "inputs larger than L2 (Q, K, V 357 MB each; prologue 1.43 GB; epilogue 4.3 GB)"},
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak, "traffic": traffic,
                     "peak_kind": f"{pk_kind} bf16 sustained (kernel inside a long step)",
                     "frac_of_nominal_2250": attn_tflops / 2250.0},
        "kernels": {"qk_norm_rope_us": statistics.mean(pro) * 1e3, "qk_norm_rope_gbs": pro_gbs,
                    "qk_norm_rope_frac_hbm": pro_gbs / pk["hbm_gbs"],
                    "varlen_attn_ms": att_ms, "varlen_attn_tflops": attn_tflops,
                    "modulate_swiglu_us": statistics.mean(epi) * 1e3, "modulate_swiglu_gbs": epi_gbs,
                    "modulate_swiglu_frac_hbm": epi_gbs / pk["hbm_gbs"], "hbm_peak_gbs": pk["hbm_gbs"],
                    "qk_norm_rope_3axis_us": rope3_us, "qk_norm_rope_3axis_gbs": rope3_gbs,
                    "qk_norm_rope_3axis_frac_hbm": rope3_gbs / pk["hbm_gbs"],
                    "qk_norm_rope_3axis_sections": list(sections),
                    "qk_norm_rope_back_to_back_us": rope1_b2b_us,
                    "qk_fullc_norm_rope_us": fullc_us, "qk_fullc_norm_rope_gbs": fullc_gbs,
                    "qk_fullc_norm_rope_frac_hbm": fullc_gbs / pk["hbm_gbs"],
                    "varlen_attn_cta_pairs": pairs,
                    "varlen_attn_skip": skip, "varlen_attn_fp8qk": fp8, "linear_epilogue": lin,
                    "bandwidth_sweep_40_heads": bw},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "graph_ms_per_step": graph_ms,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_linear_sweep(args):
    """The block's three linear layers with fused epilogues, alone, against
    cuBLAS plus torch epilogues, on the 4,096- and 58,048-token widths and on
    the 40-head sweep widths (hidden 5,120, FFN 13,824) at its four token
    counts. Activations are drawn on the device (torch's CUDA generator,
    N(0, 1), seeded per shape) to keep the multi-GB inputs off the host;
    weights as in the step."""
    import torch
    from packed_attention_qk_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    pk, pk_kind = peaks()
    shapes = [(4096, 16, 2048, 5632), (58048, 24, 3072, 8192)] + [(T, 40, 5120, 13824) for T in wl.C5_TOKENS]
    for T, H, Cd, F in shapes:
        gen = torch.Generator(device=dev)
        gen.manual_seed(T * 7 + Cd * 3 + F)

        def randn(*shape, scale=1.0, dtype=torch.bfloat16):
            return (torch.randn(*shape, generator=gen, device=dev) * scale).to(dtype)

        w = wl.Workload(f"linear layers, {T} tokens, hidden {Cd}, ffn {F}", 5, [T], H=H, D=Cd // H, C=Cd, F=F,
                        pos_runs=[[T]])
        d = {"x": randn(T, Cd), "gate_res": randn(1, Cd, scale=0.1, dtype=torch.float32),
             "cu": torch.tensor([0, T], dtype=torch.int32, device=dev)}
        o = {"o": randn(T, H, Cd // H), "h": randn(T, Cd), "act": randn(T, F)}
        res = time_linear_layers(w, d, o, pk, pk_kind)
        print(json.dumps({"sweep": "linear_epilogue", "tokens": T, "hidden": Cd, "ffn": F, **res}), flush=True)
        del d, o
        torch.cuda.empty_cache()


def run_sweep(args):
    """The HBM-bound kernels alone on the sweep shapes, one launch at a time
    with a 256 MB L2 flush in between (the 4,096-token working set is close
    to the 126 MB L2: 256 MB written, then 256 MB read, so no dirty lines are
    written back during the kernel), median of the timed launches."""
    import torch
    from packed_attention_qk_b200 import pqk
    from packed_attention_qk_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clean = torch.ones(64 << 20, dtype=torch.int32, device=dev)
    pk, pk_kind = peaks()

    def dev16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    def timed(fn, reps):
        ts = []
        for i in range(args.warmup + reps):
            flush.fill_(i & 0xFF)
            clean.sum()  # evicts the written lines before the kernel starts
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    for T in wl.C5_TOKENS:
        w = wl.config(5, T)
        p = wl.prologue_inputs(w)
        q, k, wq, wk = dev16(p["q"]), dev16(p["k"]), dev16(p["w_q"]), dev16(p["w_k"])
        pos = torch.from_numpy(p["pos"]).to(dev)
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        ms = timed(lambda: pqk.qk_norm_rope(q, k, wq, wk, pos, eps=w.eps, q_out=qo, k_out=ko), args.steps)
        gbs = w.prologue_bytes() / (ms * 1e-3) / 1e9
        print(json.dumps({"sweep": "qk_norm_rope", "tokens": T, "heads": w.H, "head_dim": w.D, "us": ms * 1e3,
                          "gbs": gbs, "frac_hbm": gbs / pk["hbm_gbs"], "peak_gbs": pk["hbm_gbs"],
                          "peak_kind": pk_kind, "bytes": w.prologue_bytes()}), flush=True)
        del q, k, qo, ko
        e = wl.epilogue_inputs(w)
        x, gate, up = dev16(e["x"]), dev16(e["gate"]), dev16(e["up"])
        shift, scale = torch.from_numpy(e["shift"]).to(dev), torch.from_numpy(e["scale"]).to(dev)
        cu = torch.from_numpy(e["cu_seqlens"]).to(dev)
        h, act = torch.empty_like(x), torch.empty_like(gate)
        ms = timed(lambda: pqk.modulate_swiglu(x, shift, scale, cu, gate=gate, up=up, eps=w.eps, h=h, act=act),
                   args.steps)
        gbs = w.epilogue_bytes() / (ms * 1e-3) / 1e9
        print(json.dumps({"sweep": "modulate_swiglu", "tokens": T, "hidden": w.C, "ffn": w.F, "us": ms * 1e3,
                          "gbs": gbs, "frac_hbm": gbs / pk["hbm_gbs"], "peak_gbs": pk["hbm_gbs"],
                          "peak_kind": pk_kind, "bytes": w.epilogue_bytes()}), flush=True)
        del x, gate, up, h, act
        torch.cuda.empty_cache()


def main():
    args = parse()
    from packed_attention_qk_b200 import workloads as wl
    if args.sweep:
        run_sweep(args)
        return
    if args.linear_sweep:
        run_linear_sweep(args)
        return
    w = wl.config(args.config)
    if args.tokens:
        w = wl.Workload(f"one request of {args.tokens} tokens, {w.H} heads x {w.D}, hidden {w.C}, ffn {w.F}", w.seed,
                        [args.tokens], H=w.H, D=w.D, C=w.C, F=w.F, pos_runs=[[args.tokens]])
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
