"""Seeded synthetic workloads for the DiT-block hot path.

This module only draws random numbers and lays out shapes. It holds none of
the hot path's arithmetic, so both the float64 oracle (tests) and the CUDA
path (library, bench) may take their inputs from it.

Workload shapes follow the serving pages' description of the problem: one
request is a joint text + audio + video token sequence of about 58k tokens
packed without padding ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长",
section "长序列注意力与通信优化"; "MiniMax H3 FastH3 real-time serving with
vLLM-Omni", section "System-wide optimizations in vLLM-Omni"). The pages give
no model dimensions; the head counts, widths and sequence mixes below are the
five stated benchmark configurations.

Recipe (every tensor has its own counter-independent stream, so a test can
draw one tensor without drawing the others):
  * stream for tensor ``name`` of config seed ``s``, chunk ``c`` =
    ``numpy.random.Generator(PCG64(SeedSequence([s, TENSOR_ID[name], c])))``,
    chunks of ``CHUNK`` elements in row-major order;
  * activations Q, K, V, x, branch, gate, up ~ N(0, 1) drawn as float32, then
    rounded once to bfloat16 (round to nearest even);
  * RMSNorm weights w_q, w_k ~ U(0.5, 1.5), rounded to bfloat16;
  * adaLN shift / scale / gated-residual gate ~ N(0, 0.1) kept in float32;
  * outlier variant: an i.i.d. Bernoulli(0.001) mask over K's elements; masked
    elements are multiplied by 20 in float32 before the bfloat16 rounding;
  * block-scaled attention inputs (key-block skipping tests): Q ~ 2.5 N(0, 1);
    K ~ N(0, 1) times a per-(request, 128-key block) factor, 3 ("strong") or
    0.02 ("weak") with probability 1/2 each from stream ``skip_blocks``;
  * local attention inputs (a stand-in for video attention, whose weight sits
    on nearby tokens): every token gets a unit feature vector of sinusoids of
    its (t, h, w) ids, Q = K-ish = A * feature + N(0, 1) noise per head;
  * linear layers around the fused operators: inputs (attention output, h,
    SwiGLU output) ~ N(0, 1); weights [out, in] ~ N(0, 1 / in) drawn as
    float32 and scaled before the one bfloat16 rounding (random
    initialisation; no trained weights exist here).
bfloat16 tensors are returned as their uint16 bit patterns.
"""

from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, field

import numpy as np

CHUNK = 1 << 22

TENSOR_ID = {
    "q": 1, "k": 2, "v": 3, "x": 4, "branch": 5, "gate": 6, "up": 7,
    "w_q": 8, "w_k": 9, "shift": 10, "scale": 11, "gate_res": 12,
    "outlier": 13, "sample_rows": 14, "w_q_full": 15, "w_k_full": 16,
    "skip_blocks": 17, "q_local": 18, "k_local": 19,
    "attn_out": 20, "w_o": 21, "h_in": 22, "w1": 23, "act_in": 24, "w2": 25,
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest even) and return the uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


def _chunk_rng(seed: int, name: str, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, TENSOR_ID[name], chunk])))


def _chunk_values(seed: int, name: str, c: int, m: int, kind: str) -> np.ndarray:
    g = _chunk_rng(seed, name, c)
    if kind == "normal":
        return g.standard_normal(m, dtype=np.float32)
    if kind == "normal01":
        return g.standard_normal(m, dtype=np.float32) * np.float32(0.1)
    if kind == "uniform_w":
        return g.uniform(0.5, 1.5, m).astype(np.float32)
    if kind == "bernoulli":
        return (g.random(m, dtype=np.float32) < np.float32(0.001)).astype(np.float32)
    raise ValueError(kind)


def _draw(seed: int, name: str, n: int, kind: str, threads: int | None = None, to_bf16: bool = False,
          outlier_name: str | None = None) -> np.ndarray:
    """Draw ``n`` values of distribution ``kind`` chunk by chunk: float32, or
    bf16 bits rounded per chunk (``to_bf16``) so that no full-size float32
    temporary exists. With ``outlier_name``, elements whose Bernoulli(0.001)
    mask (stream ``outlier_name``) is set are multiplied by 20 first."""
    out = np.empty(n, dtype=np.uint16 if to_bf16 else np.float32)
    nchunks = (n + CHUNK - 1) // CHUNK

    def fill(c: int) -> None:
        lo, hi = c * CHUNK, min(n, (c + 1) * CHUNK)
        vals = _chunk_values(seed, name, c, hi - lo, kind)
        if outlier_name is not None:
            m = _chunk_values(seed, outlier_name, c, hi - lo, "bernoulli")
            vals = np.where(m > 0, vals * np.float32(20.0), vals)
        out[lo:hi] = f32_to_bf16_bits(vals) if to_bf16 else vals

    if nchunks <= 1:
        if nchunks:
            fill(0)
        return out
    nt = threads or min(16, os.cpu_count() or 1)
    with _cf.ThreadPoolExecutor(nt) as ex:
        list(ex.map(fill, range(nchunks)))
    return out


def bf16_normal(seed: int, name: str, shape: tuple[int, ...]) -> np.ndarray:
    n = int(np.prod(shape))
    return _draw(seed, name, n, "normal", to_bf16=True).reshape(shape)


def bf16_weight(seed: int, name: str, d: int) -> np.ndarray:
    return f32_to_bf16_bits(_draw(seed, name, d, "uniform_w"))


def f32_modulation(seed: int, name: str, shape: tuple[int, ...]) -> np.ndarray:
    n = int(np.prod(shape))
    return _draw(seed, name, n, "normal01").reshape(shape)


def bf16_k_with_outliers(seed: int, shape: tuple[int, ...]) -> np.ndarray:
    """K for the outlier variant: 0.1% of entries multiplied by 20 before rounding."""
    n = int(np.prod(shape))
    return _draw(seed, "k", n, "normal", to_bf16=True, outlier_name="outlier").reshape(shape)


# ----------------------------------------------------------------------------
# Configurations
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    seed: int
    seg_lens: list[int]
    H: int
    D: int
    C: int
    F: int
    # positions of each segment as a list of (modality, length) runs; ids
    # restart at 0 for each run
    pos_runs: list[list[int]] = field(default_factory=list)
    rope_base: float = 10000.0
    eps: float = 1e-6
    attention: bool = True

    @property
    def T(self) -> int:
        return int(sum(self.seg_lens))

    @property
    def B(self) -> int:
        return len(self.seg_lens)

    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seg_lens)]).astype(np.int32)

    def positions(self) -> np.ndarray:
        """Per-token RoPE ids; they restart at 0 for each modality run."""
        parts = []
        for runs in self.pos_runs:
            for n in runs:
                parts.append(np.arange(n, dtype=np.int32))
        p = np.concatenate(parts) if parts else np.zeros(0, np.int32)
        assert p.shape[0] == self.T
        return p

    def positions3(self, video_grid: tuple[int, int, int] = (12, 48, 96)) -> np.ndarray:
        """[T, 3] (t, h, w) ids for the three-axis RoPE variant: a modality
        run whose length equals the video latent grid gets the grid's
        (t, h, w) coordinates in token order (t-major); every other run gets
        its one-axis ids repeated on the three axes."""
        nt, nh, nw = video_grid
        parts = []
        for runs in self.pos_runs:
            for n in runs:
                if n == nt * nh * nw:
                    t, h, w = np.meshgrid(np.arange(nt), np.arange(nh), np.arange(nw), indexing="ij")
                    parts.append(np.stack([t.ravel(), h.ravel(), w.ravel()], 1))
                else:
                    a = np.arange(n)
                    parts.append(np.stack([a, a, a], 1))
        p = np.concatenate(parts).astype(np.int32) if parts else np.zeros((0, 3), np.int32)
        assert p.shape[0] == self.T
        return np.ascontiguousarray(p)

    def attn_flops(self) -> float:
        """4*H*D per valid (query, key) pair within a request."""
        return 4.0 * self.H * self.D * float(sum(int(L) * int(L) for L in self.seg_lens))

    def prologue_bytes(self, three_axis: bool = False) -> int:
        """qk_norm_rope: Q and K read + written (bf16) plus the int32
        position (three of them for the (t, h, w) variant)."""
        return self.T * (8 * self.H * self.D + (12 if three_axis else 4))

    def epilogue_bytes(self, with_branch: bool = False) -> int:
        """modulate_swiglu: x (+branch, +x_out) in, h out; gate, up in; act out."""
        per_tok = 2 * (2 * self.C + 3 * self.F) if not with_branch else 2 * (4 * self.C + 3 * self.F)
        return self.T * per_tok


def _c1() -> Workload:
    return Workload("tiny packed attention block: 2 sequences 200+312 tokens, 4 heads, head_dim 64",
                    0, [200, 312], H=4, D=64, C=256, F=512, pos_runs=[[200], [312]])


def _c2() -> Workload:
    return Workload("joint sequence of 4,096 tokens (text 256 + audio 512 + video 3,328), 16 heads, head_dim 128",
                    1, [4096], H=16, D=128, C=2048, F=5632, pos_runs=[[256, 512, 3328]])


def _c3() -> Workload:
    # video tokens: 12 latent frames x 48 x 96; the flattened (t, h, w) id in
    # token order is t*48*96 + h*96 + w, i.e. 0..55,295
    return Workload("joint sequence of 58,048 tokens (text 512 + audio 2,240 + video 12x48x96), 24 heads, head_dim 128",
                    2, [58048], H=24, D=128, C=3072, F=8192, pos_runs=[[512, 2240, 55296]])


def _c4() -> Workload:
    lens = [12345, 29024, 58048, 87072]
    runs = [[12345], [29024], [512, 2240, 55296], [87072]]
    return Workload("varlen batch of 4 requests 12,345/29,024/58,048/87,072 tokens, 24 heads, head_dim 128",
                    3, lens, H=24, D=128, C=3072, F=8192, pos_runs=runs)


def _c5(T: int) -> Workload:
    return Workload(f"prologue/epilogue bandwidth sweep, {T} tokens, 40 heads x 128, hidden 5,120, ffn 13,824",
                    4, [T], H=40, D=128, C=5120, F=13824, pos_runs=[[T]], attention=False)


C5_TOKENS = (4096, 16384, 58048, 186489)


def config(i: int, t5: int = 58048) -> Workload:
    """The five benchmark configurations, 1-based like their numbering."""
    if i == 1:
        return _c1()
    if i == 2:
        return _c2()
    if i == 3:
        return _c3()
    if i == 4:
        return _c4()
    if i == 5:
        return _c5(t5)
    raise ValueError(i)


def custom(seg_lens: list[int], H: int, D: int, C: int | None = None, F: int | None = None,
           seed: int = 100) -> Workload:
    """Small ad-hoc shapes for edge-case tests; positions 0..L-1 per segment."""
    C = C if C is not None else H * D
    F = F if F is not None else 2 * C
    return Workload(f"custom {seg_lens} H{H} D{D}", seed, list(seg_lens), H=H, D=D, C=C, F=F,
                    pos_runs=[[L] for L in seg_lens])


# ----------------------------------------------------------------------------
# Tensor sets
# ----------------------------------------------------------------------------

def attention_inputs(w: Workload, outliers: bool = False) -> dict[str, np.ndarray]:
    shp = (w.T, w.H, w.D)
    k = bf16_k_with_outliers(w.seed, shp) if outliers else bf16_normal(w.seed, "k", shp)
    return {"q": bf16_normal(w.seed, "q", shp), "k": k, "v": bf16_normal(w.seed, "v", shp),
            "cu_seqlens": w.cu_seqlens()}


def prologue_inputs(w: Workload) -> dict[str, np.ndarray]:
    shp = (w.T, w.H, w.D)
    return {"q": bf16_normal(w.seed, "q", shp), "k": bf16_normal(w.seed, "k", shp),
            "w_q": bf16_weight(w.seed, "w_q", w.D), "w_k": bf16_weight(w.seed, "w_k", w.D),
            "pos": w.positions()}


def fullc_weights(w: Workload) -> dict[str, np.ndarray]:
    """Weights of the full-width Q/K norm: one per element of the H*D row."""
    return {"w_q": bf16_weight(w.seed, "w_q_full", w.H * w.D), "w_k": bf16_weight(w.seed, "w_k_full", w.H * w.D)}


def epilogue_inputs(w: Workload, with_branch: bool = False) -> dict[str, np.ndarray]:
    d = {"x": bf16_normal(w.seed, "x", (w.T, w.C)),
         "gate": bf16_normal(w.seed, "gate", (w.T, w.F)),
         "up": bf16_normal(w.seed, "up", (w.T, w.F)),
         "shift": f32_modulation(w.seed, "shift", (w.B, w.C)),
         "scale": f32_modulation(w.seed, "scale", (w.B, w.C)),
         "gate_res": f32_modulation(w.seed, "gate_res", (w.B, w.C)),
         "cu_seqlens": w.cu_seqlens()}
    if with_branch:
        d["branch"] = bf16_normal(w.seed, "branch", (w.T, w.C))
    return d


def block_scaled_attention_inputs(w: Workload, strong: float = 3.0, weak: float = 0.02,
                                  q_scale: float = 2.5) -> dict[str, np.ndarray]:
    """Q ~ q_scale N(0, 1); K ~ N(0, 1) times a factor per (request, block of
    128 keys counted from the request's first token), ``strong`` or ``weak``
    with probability 1/2 each; V ~ N(0, 1). Returns bf16 bits plus the block
    factors (one per block, requests in order)."""
    shp = (w.T, w.H, w.D)
    n = w.T * w.H * w.D
    cu = w.cu_seqlens()
    nblk = [(int(L) + 127) // 128 for L in w.seg_lens]
    g = _chunk_rng(w.seed, "skip_blocks", 0)
    factors = np.where(g.random(int(sum(nblk))) < 0.5, weak, strong).astype(np.float32)
    per_key = np.empty(w.T, np.float32)
    b0 = 0
    for i, L in enumerate(w.seg_lens):
        lo = int(cu[i])
        for j in range(nblk[i]):
            per_key[lo + 128 * j: lo + min(int(L), 128 * (j + 1))] = factors[b0 + j]
        b0 += nblk[i]
    q = f32_to_bf16_bits(_draw(w.seed, "q", n, "normal").reshape(shp) * np.float32(q_scale))
    k = f32_to_bf16_bits(_draw(w.seed, "k", n, "normal").reshape(shp) * per_key[:, None, None])
    return {"q": q, "k": k, "v": bf16_normal(w.seed, "v", shp), "cu_seqlens": cu, "block_factors": factors}


def local_features(pos3: np.ndarray, D: int, base: float = 100.0) -> np.ndarray:
    """[T, D] unit vectors of sinusoids of the (t, h, w) ids: D/8 frequency
    pairs for t, 3D/16 each for h and w, frequencies base^(-i/n) per axis;
    the inner product of two tokens' vectors is the mean over pairs of
    cos(id difference * frequency)."""
    n_axis = (D // 8, 3 * D // 16, 3 * D // 16)
    assert sum(n_axis) * 2 == D
    cols = []
    for a, n in enumerate(n_axis):
        freq = base ** (-np.arange(n) / n)
        ang = pos3[:, a:a + 1].astype(np.float64) * freq[None, :]
        cols += [np.cos(ang), np.sin(ang)]
    f = np.concatenate(cols, axis=1) / np.sqrt(D / 2)
    return f.astype(np.float32)


def local_attention_inputs(w: Workload, amplitude: float = 12.0, noise: float = 1.0,
                           video_grid: tuple[int, int, int] = (12, 48, 96)) -> dict[str, np.ndarray]:
    """Q[t, h] = amplitude * f(t) + noise * N(0, 1), K the same with its own
    noise, V ~ N(0, 1); f = local_features of the (t, h, w) ids (positions3).
    Drawn head by head (stream chunk = head index) to bound host memory."""
    f = local_features(w.positions3(video_grid), w.D) * np.float32(amplitude)
    q = np.empty((w.T, w.H, w.D), np.uint16)
    k = np.empty((w.T, w.H, w.D), np.uint16)

    def head(h: int) -> None:
        for name, out in (("q_local", q), ("k_local", k)):
            z = _chunk_rng(w.seed, name, h).standard_normal((w.T, w.D), dtype=np.float32)
            out[:, h, :] = f32_to_bf16_bits(f + np.float32(noise) * z)

    with _cf.ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(head, range(w.H)))
    return {"q": q, "k": k, "v": bf16_normal(w.seed, "v", (w.T, w.H, w.D)), "cu_seqlens": w.cu_seqlens()}


def bf16_linear_weight(seed: int, name: str, n_out: int, n_in: int) -> np.ndarray:
    """[n_out, n_in] weight ~ N(0, 1 / n_in), rounded once to bfloat16."""
    scale = np.float32(1.0 / np.sqrt(n_in))
    out = np.empty(n_out * n_in, np.uint16)
    for c in range((n_out * n_in + CHUNK - 1) // CHUNK):
        lo, hi = c * CHUNK, min(n_out * n_in, (c + 1) * CHUNK)
        out[lo:hi] = f32_to_bf16_bits(_chunk_values(seed, name, c, hi - lo, "normal") * scale)
    return out.reshape(n_out, n_in)


def linear_inputs(w: Workload, which: str) -> dict[str, np.ndarray]:
    """Operands of one linear layer of the block, bf16 bits:
    ``"o_proj"``: a = attention output [T, C], w = W_o [C, C], plus x, gate_res
    for the gated residual; ``"w1"``: a = h [T, C], w = W1 [2F, C] (gate rows,
    then up rows); ``"w2"``: a = SwiGLU output [T, F], w = W2 [C, F], plus x,
    gate_res."""
    T, Cd, F = w.T, w.C, w.F
    if which == "o_proj":
        d = {"a": bf16_normal(w.seed, "attn_out", (T, Cd)), "w": bf16_linear_weight(w.seed, "w_o", Cd, Cd)}
    elif which == "w1":
        return {"a": bf16_normal(w.seed, "h_in", (T, Cd)), "w": bf16_linear_weight(w.seed, "w1", 2 * F, Cd)}
    elif which == "w2":
        d = {"a": bf16_normal(w.seed, "act_in", (T, F)), "w": bf16_linear_weight(w.seed, "w2", Cd, F)}
    else:
        raise ValueError(which)
    d["x"] = bf16_normal(w.seed, "x", (T, Cd))
    d["gate_res"] = f32_modulation(w.seed, "gate_res", (w.B, Cd))
    d["cu_seqlens"] = w.cu_seqlens()
    return d


def sample_rows(w: Workload, per_segment: int = 256) -> np.ndarray:
    """Seeded query-row sample: per segment, its first and last row plus
    ``per_segment - 2`` distinct rows drawn with seed (config seed + 1000)."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed + 1000, TENSOR_ID["sample_rows"]])))
    cu = w.cu_seqlens()
    rows = []
    for i in range(w.B):
        lo, hi = int(cu[i]), int(cu[i + 1])
        L = hi - lo
        if L == 0:
            continue
        if L <= per_segment:
            rows.append(np.arange(lo, hi))
            continue
        mid = g.choice(np.arange(lo + 1, hi - 1), size=per_segment - 2, replace=False)
        rows.append(np.sort(np.concatenate([[lo], mid, [hi - 1]])))
    return np.concatenate(rows).astype(np.int32) if rows else np.zeros(0, np.int32)
