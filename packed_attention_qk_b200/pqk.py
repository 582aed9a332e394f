"""Thin Python binding of libpqk's C ABI (include/pqk.h).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels behind the C ABI. PyTorch supplies device memory (``data_ptr``) and
the current CUDA stream. There is no fallback: if ``libpqk.so`` has not been
built, loading fails with an error.
"""

from __future__ import annotations

import ctypes as C
import math
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpqk.so")

PQK_OK = 0
STATUS = {0: "PQK_OK", -1: "PQK_ERR_INVALID_ARG", -2: "PQK_ERR_UNSUPPORTED", -3: "PQK_ERR_MISALIGNED",
          -4: "PQK_ERR_CUDA", -5: "PQK_ERR_WORKSPACE", -6: "PQK_ERR_TIMEOUT", -7: "PQK_ERR_BAD_SEQLENS"}
ROPE_INTERLEAVED, ROPE_HALF = 0, 1
NORM_RMS, NORM_LAYER, NORM_NONE = 0, 1, 2

# every symbol include/pqk.h declares
EXPORTS = ("pqk_qk_norm_rope", "pqk_qk_norm_rope_e4m3", "pqk_qk_norm_rope_3axis", "pqk_qk_fullc_norm_rope", "pqk_varlen_attn_workspace_size", "pqk_varlen_attn_fwd",
           "pqk_varlen_attn_fwd_skip", "pqk_quantize_qk_e4m3", "pqk_varlen_attn_fwd_fp8qk", "pqk_quantize_e4m3",
           "pqk_varlen_attn_fwd_fp8",
           "pqk_varlen_attn_fwd_noalloc", "pqk_modulate_swiglu", "pqk_linear_gated_residual", "pqk_linear_swiglu",
           "pqk_get_device_status", "pqk_set_wait_timeout_ns", "pqk_set_attn_cta_pairs", "pqk_selftest_wait_timeout",
           "pqk_status_string",
           "pqk_version")


class PqkError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code} ({STATUS.get(code, 'unknown')}: {status_string(code)})")
        self.code = code


_lib = None


def lib(path: str | None = None) -> C.CDLL:
    """Load libpqk.so (built by packed_attention_qk_b200.build) and declare
    its signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libpqk.so not found at {p}: build it with `python -m packed_attention_qk_b200.build`")
    L = C.CDLL(p)
    vp, i64, i32, f32, sz = C.c_void_p, C.c_int64, C.c_int, C.c_float, C.c_size_t
    L.pqk_qk_norm_rope.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, vp, vp, vp, i64, i32, i32, f32, f32, i32, vp]
    L.pqk_qk_norm_rope.restype = i32
    L.pqk_qk_norm_rope_e4m3.argtypes = [vp, vp, vp, vp, i64, i64, vp, vp, vp, i64, i32, i32, f32, f32, i32, vp, vp]
    L.pqk_qk_norm_rope_e4m3.restype = i32
    L.pqk_qk_norm_rope_3axis.argtypes = [vp, vp, vp, vp, i64, i64, vp, vp, vp, i32, i32, i32, i64, i32, i32, f32, f32,
                                         i32, vp]
    L.pqk_qk_norm_rope_3axis.restype = i32
    L.pqk_qk_fullc_norm_rope.argtypes = [vp, vp, vp, vp, i64, i64, vp, vp, vp, i64, i32, i32, f32, f32, i32, vp]
    L.pqk_qk_fullc_norm_rope.restype = i32
    L.pqk_varlen_attn_workspace_size.argtypes = [i32]
    L.pqk_varlen_attn_workspace_size.restype = sz
    L.pqk_varlen_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i32, i64, i32, i32, f32, vp, sz,
                                      vp]
    L.pqk_varlen_attn_fwd.restype = i32
    L.pqk_varlen_attn_fwd_skip.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i32, i64, i32, i32, f32, f32,
                                           vp, vp, sz, vp]
    L.pqk_varlen_attn_fwd_skip.restype = i32
    L.pqk_quantize_qk_e4m3.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp]
    L.pqk_quantize_qk_e4m3.restype = i32
    L.pqk_varlen_attn_fwd_fp8qk.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, vp, i32, i64, i32, i32, f32, f32, vp,
                                            vp, sz, vp]
    L.pqk_varlen_attn_fwd_fp8qk.restype = i32
    L.pqk_quantize_e4m3.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp]
    L.pqk_quantize_e4m3.restype = i32
    L.pqk_varlen_attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp, i32, i64, i32, i32, f32, f32, vp, vp, sz,
                                          vp]
    L.pqk_varlen_attn_fwd_fp8.restype = i32
    L.pqk_varlen_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i32, i64, i32, i32, f32,
                                              vp]
    L.pqk_varlen_attn_fwd_noalloc.restype = i32
    L.pqk_modulate_swiglu.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, f32, vp, vp, i64, vp,
                                      i32, vp]
    L.pqk_modulate_swiglu.restype = i32
    L.pqk_linear_gated_residual.argtypes = [vp, i64, vp, vp, i64, vp, vp, i32, vp, i64, i64, i32, i32, vp]
    L.pqk_linear_gated_residual.restype = i32
    L.pqk_linear_swiglu.argtypes = [vp, i64, vp, vp, i64, i64, i32, i32, vp]
    L.pqk_linear_swiglu.restype = i32
    L.pqk_get_device_status.argtypes = [vp]
    L.pqk_get_device_status.restype = i32
    L.pqk_set_wait_timeout_ns.argtypes = [i64]
    L.pqk_set_wait_timeout_ns.restype = None
    L.pqk_set_attn_cta_pairs.argtypes = [C.c_int]
    L.pqk_set_attn_cta_pairs.restype = None
    L.pqk_selftest_wait_timeout.argtypes = [i64, vp]
    L.pqk_selftest_wait_timeout.restype = i32
    L.pqk_status_string.argtypes = [i32]
    L.pqk_status_string.restype = C.c_char_p
    L.pqk_version.argtypes = []
    L.pqk_version.restype = C.c_char_p
    if path is None:
        _lib = L
    return L


def status_string(code: int) -> str:
    return lib().pqk_status_string(code).decode()


def _check(fn: str, rc: int) -> None:
    if rc != PQK_OK:
        raise PqkError(fn, rc)


def _stream(stream) -> int | None:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _token_stride(t, ndim: int) -> int:
    assert t.dim() == ndim, f"expected a {ndim}-d tensor, got {tuple(t.shape)}"
    for d in range(1, ndim):
        want = 1
        for e in range(d + 1, ndim):
            want *= t.shape[e]
        assert t.stride(d) == want, "only the token (first) dimension may be strided"
    return t.stride(0)


# ---------------------------------------------------------------- calls

def qk_norm_rope(q, k, w_q, w_k, pos, *, eps: float = 1e-6, rope_base: float = 10000.0,
                 style: int = ROPE_INTERLEAVED, q_out=None, k_out=None, stream=None):
    """Fused Q/K RMSNorm + RoPE. q, k: bf16 [T, H, D] (token dim may be
    strided); q_out, k_out: [T, H, D] views with their own token strides
    (default: in place)."""
    q_out = q if q_out is None else q_out
    k_out = k if k_out is None else k_out
    T, H, D = q.shape
    assert tuple(q_out.shape) == (T, H, D) and tuple(k_out.shape) == (T, H, D)
    _check("pqk_qk_norm_rope", lib().pqk_qk_norm_rope(
        _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _token_stride(q, 3), _token_stride(k, 3), _token_stride(q_out, 3),
        _token_stride(k_out, 3), _ptr(w_q), _ptr(w_k), _ptr(pos), T, H, D, eps, rope_base, style, _stream(stream)))
    return q_out, k_out


def qk_norm_rope_e4m3(q, k, w_q, w_k, pos, *, eps: float = 1e-6, rope_base: float = 10000.0,
                      style: int = ROPE_INTERLEAVED, q8=None, k8=None, deq=None, stream=None):
    """Fused Q/K RMSNorm + RoPE with e4m3 output at the per-tensor bound
    scale sqrt(D) max|w| -> 448. Returns (q8, k8 uint8 [T, H, D], deq fp32 [2H])."""
    import torch
    T, H, D = q.shape
    if q8 is None:
        q8 = torch.empty((T, H, D), dtype=torch.uint8, device=q.device)
    if k8 is None:
        k8 = torch.empty((T, H, D), dtype=torch.uint8, device=q.device)
    if deq is None:
        deq = torch.empty(2 * H, dtype=torch.float32, device=q.device)
    assert q8.is_contiguous() and k8.is_contiguous() and deq.numel() >= 2 * H
    _check("pqk_qk_norm_rope_e4m3", lib().pqk_qk_norm_rope_e4m3(
        _ptr(q), _ptr(k), _ptr(q8), _ptr(k8), _token_stride(q, 3), _token_stride(k, 3), _ptr(w_q), _ptr(w_k),
        _ptr(pos), T, H, D, eps, rope_base, style, _ptr(deq), _stream(stream)))
    return q8, k8, deq


def qk_norm_rope_3axis(q, k, w_q, w_k, pos3, sections, *, eps: float = 1e-6, rope_base: float = 10000.0,
                       style: int = ROPE_INTERLEAVED, q_out=None, k_out=None, stream=None):
    """Fused Q/K RMSNorm + RoPE with (t, h, w) ids per token (pos3: int32
    [T, 3]); sections: pairs per axis, summing to D/2."""
    q_out = q if q_out is None else q_out
    k_out = k if k_out is None else k_out
    T, H, D = q.shape
    qs, ks = _token_stride(q, 3), _token_stride(k, 3)
    assert _token_stride(q_out, 3) == qs and _token_stride(k_out, 3) == ks
    st, sh, sw = (int(v) for v in sections)
    _check("pqk_qk_norm_rope_3axis", lib().pqk_qk_norm_rope_3axis(
        _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), qs, ks, _ptr(w_q), _ptr(w_k), _ptr(pos3), st, sh, sw, T, H, D,
        eps, rope_base, style, _stream(stream)))
    return q_out, k_out


def qk_fullc_norm_rope(q, k, w_q, w_k, pos, *, eps: float = 1e-6, rope_base: float = 10000.0,
                       style: int = ROPE_INTERLEAVED, q_out=None, k_out=None, stream=None):
    """Fused Q/K RMSNorm over all H*D elements of a token (weights [H*D]) +
    RoPE per head."""
    q_out = q if q_out is None else q_out
    k_out = k if k_out is None else k_out
    T, H, D = q.shape
    qs, ks = _token_stride(q, 3), _token_stride(k, 3)
    assert _token_stride(q_out, 3) == qs and _token_stride(k_out, 3) == ks
    _check("pqk_qk_fullc_norm_rope", lib().pqk_qk_fullc_norm_rope(
        _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), qs, ks, _ptr(w_q), _ptr(w_k), _ptr(pos), T, H, D, eps,
        rope_base, style, _stream(stream)))
    return q_out, k_out


def varlen_attn_workspace_size(B: int) -> int:
    return int(lib().pqk_varlen_attn_workspace_size(B))


def varlen_attn_fwd(q, k, v, cu_seqlens, *, softmax_scale: float | None = None, o=None, lse=None,
                    workspace=None, want_lse: bool = False, stream=None):
    """Packed varlen attention. q, k, v: bf16 [T, H, D]; cu_seqlens: int32
    [B+1] on the device. Returns (o, lse or None)."""
    import torch
    T, H, D = q.shape
    B = cu_seqlens.shape[0] - 1
    scale = softmax_scale if softmax_scale is not None else D ** -0.5
    if o is None:
        o = torch.empty((T, H, D), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((H, T), dtype=torch.float32, device=q.device)
    ws_bytes = varlen_attn_workspace_size(B)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _check("pqk_varlen_attn_fwd", lib().pqk_varlen_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _token_stride(q, 3), _token_stride(k, 3),
        _token_stride(v, 3), _token_stride(o, 3), _ptr(cu_seqlens), B, T, H, D, scale, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return o, lse


def varlen_attn_fwd_skip(q, k, v, cu_seqlens, skip_threshold_log2: float, *, softmax_scale: float | None = None,
                         o=None, lse=None, workspace=None, want_lse: bool = False, skip_counts=None, stream=None):
    """Packed varlen attention that drops key blocks whose scores lie more
    than skip_threshold_log2 (log2 units) below the earlier blocks' maximum
    for every row of a 32-row query block. skip_counts: None or a device
    int64 tensor of 2 elements that the call adds to (dropped 32-row blocks,
    left-out 128-row P x V products). Returns (o, lse or None)."""
    import torch
    T, H, D = q.shape
    B = cu_seqlens.shape[0] - 1
    scale = softmax_scale if softmax_scale is not None else D ** -0.5
    if o is None:
        o = torch.empty((T, H, D), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((H, T), dtype=torch.float32, device=q.device)
    ws_bytes = varlen_attn_workspace_size(B)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if skip_counts is not None:
        assert skip_counts.dtype == torch.int64 and skip_counts.numel() >= 2 and skip_counts.is_contiguous()
    _check("pqk_varlen_attn_fwd_skip", lib().pqk_varlen_attn_fwd_skip(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _token_stride(q, 3), _token_stride(k, 3),
        _token_stride(v, 3), _token_stride(o, 3), _ptr(cu_seqlens), B, T, H, D, scale, float(skip_threshold_log2),
        _ptr(skip_counts), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return o, lse


def quantize_qk_e4m3(q, k, *, q8=None, k8=None, scales=None, stream=None):
    """Per-head absmax e4m3 quantisation of Q and K (bf16 [T, H, D]).
    Returns (q8, k8 uint8 [T, H, D], deq fp32 [2H] view of ``scales``)."""
    import torch
    T, H, D = q.shape
    if q8 is None:
        q8 = torch.empty((T, H, D), dtype=torch.uint8, device=q.device)
    if k8 is None:
        k8 = torch.empty((T, H, D), dtype=torch.uint8, device=q.device)
    if scales is None:
        scales = torch.empty(4 * H, dtype=torch.float32, device=q.device)
    assert q8.is_contiguous() and k8.is_contiguous() and scales.numel() >= 4 * H
    _check("pqk_quantize_qk_e4m3", lib().pqk_quantize_qk_e4m3(
        _ptr(q), _ptr(k), _token_stride(q, 3), _token_stride(k, 3), T, H, D, _ptr(q8), _ptr(k8), _ptr(scales),
        _stream(stream)))
    return q8, k8, scales[2 * H:4 * H]


def varlen_attn_fwd_fp8qk(q8, k8, v, deq, cu_seqlens, *, softmax_scale: float | None = None, o=None, lse=None,
                          workspace=None, want_lse: bool = False, skip_threshold_log2: float = math.inf,
                          skip_counts=None, stream=None):
    """Packed varlen attention with Q K^T on the FP8 tensor cores: q8, k8
    e4m3 bytes [T, H, D] (quantize_qk_e4m3), deq fp32 [2H], v bf16; block
    skipping as varlen_attn_fwd_skip when skip_threshold_log2 is finite.
    Returns (o, lse or None)."""
    import torch
    T, H, D = v.shape
    B = cu_seqlens.shape[0] - 1
    scale = softmax_scale if softmax_scale is not None else D ** -0.5
    if o is None:
        o = torch.empty((T, H, D), dtype=v.dtype, device=v.device)
    if lse is None and want_lse:
        lse = torch.empty((H, T), dtype=torch.float32, device=v.device)
    if workspace is None:
        workspace = torch.empty(varlen_attn_workspace_size(B), dtype=torch.uint8, device=v.device)
    assert q8.is_contiguous() and k8.is_contiguous() and tuple(q8.shape) == (T, H, D) == tuple(k8.shape)
    _check("pqk_varlen_attn_fwd_fp8qk", lib().pqk_varlen_attn_fwd_fp8qk(
        _ptr(q8), _ptr(k8), _ptr(v), _ptr(deq), _ptr(o), _ptr(lse), _token_stride(v, 3), _token_stride(o, 3),
        _ptr(cu_seqlens), B, T, H, D, scale, float(skip_threshold_log2), _ptr(skip_counts), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return o, lse


def quantize_e4m3(x, *, x8=None, scales=None, stream=None):
    """Per-head absmax e4m3 quantisation of one bf16 [T, H, D] tensor.
    Returns (x8 uint8 [T, H, D], deq fp32 [H] view of ``scales``)."""
    import torch
    T, H, D = x.shape
    if x8 is None:
        x8 = torch.empty((T, H, D), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(2 * H, dtype=torch.float32, device=x.device)
    assert x8.is_contiguous() and scales.numel() >= 2 * H
    _check("pqk_quantize_e4m3", lib().pqk_quantize_e4m3(_ptr(x), _token_stride(x, 3), T, H, D, _ptr(x8),
                                                         _ptr(scales), _stream(stream)))
    return x8, scales[H:2 * H]


def varlen_attn_fwd_fp8(q8, k8, v8, deq, cu_seqlens, *, softmax_scale: float | None = None, o=None, lse=None,
                        workspace=None, want_lse: bool = False, skip_threshold_log2: float = math.inf,
                        skip_counts=None, stream=None):
    """The attention with Q K^T and P V on the FP8 tensor cores: q8, k8, v8
    e4m3 bytes [T, H, D]; deq fp32 [3H] (Q's, K's, V's factors). A finite
    skip_threshold_log2 adds block skipping (skip_counts as in
    varlen_attn_fwd_skip). Returns (o bf16 [T, H, D], lse or None)."""
    import torch
    T, H, D = q8.shape
    B = cu_seqlens.shape[0] - 1
    scale = softmax_scale if softmax_scale is not None else D ** -0.5
    if o is None:
        o = torch.empty((T, H, D), dtype=torch.bfloat16, device=q8.device)
    if lse is None and want_lse:
        lse = torch.empty((H, T), dtype=torch.float32, device=q8.device)
    if workspace is None:
        workspace = torch.empty(varlen_attn_workspace_size(B), dtype=torch.uint8, device=q8.device)
    for t in (q8, k8, v8):
        assert t.is_contiguous() and tuple(t.shape) == (T, H, D)
    assert deq.is_contiguous() and deq.numel() >= 3 * H
    if skip_counts is not None:
        assert skip_counts.dtype == torch.int64 and skip_counts.numel() >= 2 and skip_counts.is_contiguous()
    _check("pqk_varlen_attn_fwd_fp8", lib().pqk_varlen_attn_fwd_fp8(
        _ptr(q8), _ptr(k8), _ptr(v8), _ptr(deq), _ptr(o), _ptr(lse), _token_stride(o, 3), _ptr(cu_seqlens), B, T, H,
        D, scale, float(skip_threshold_log2), _ptr(skip_counts), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return o, lse


def varlen_attn_fwd_noalloc(q, k, v, cu_seqlens, *, softmax_scale: float | None = None, o=None, lse=None,
                            want_lse: bool = False, stream=None):
    """Packed varlen attention for callers that cannot allocate device
    memory: the tile schedule lives in the library's own fixed device array
    (at most 4096 requests; calls must not overlap on the GPU). The outputs
    are allocated here only when not passed in."""
    import torch
    T, H, D = q.shape
    B = cu_seqlens.shape[0] - 1
    scale = softmax_scale if softmax_scale is not None else D ** -0.5
    if o is None:
        o = torch.empty((T, H, D), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((H, T), dtype=torch.float32, device=q.device)
    _check("pqk_varlen_attn_fwd_noalloc", lib().pqk_varlen_attn_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _token_stride(q, 3), _token_stride(k, 3),
        _token_stride(v, 3), _token_stride(o, 3), _ptr(cu_seqlens), B, T, H, D, scale, _stream(stream)))
    return o, lse


def modulate_swiglu(x, shift, scale, cu_seqlens, *, gate_res=None, branch=None, gate=None, up=None,
                    norm_type: int = NORM_RMS, eps: float = 1e-6, x_out=None, h=None, act=None, stream=None):
    """Fused gated residual + norm + adaLN modulation, and SwiGLU.
    Returns (x_out or None, h, act or None)."""
    import torch
    T, Cdim = x.shape
    B = cu_seqlens.shape[0] - 1
    if h is None:
        h = torch.empty_like(x)
    F, gu_stride = 0, 0
    if gate is not None:
        F = gate.shape[1]
        gu_stride = _token_stride(gate, 2)
        assert _token_stride(up, 2) == gu_stride
        if act is None:
            act = torch.empty((T, F), dtype=x.dtype, device=x.device)
    _check("pqk_modulate_swiglu", lib().pqk_modulate_swiglu(
        _ptr(x), _ptr(branch), _ptr(x_out), _ptr(h), _ptr(shift), _ptr(scale), _ptr(gate_res), _ptr(cu_seqlens),
        B, T, Cdim, norm_type, eps, _ptr(gate), _ptr(up), gu_stride, _ptr(act), F, _stream(stream)))
    return x_out, h, act


def linear_gated_residual(a, w, *, x=None, gate_res=None, cu_seqlens=None, out=None, stream=None):
    """out = x + gate_res[request] * (a @ w.T) on the tensor cores (the
    residual add in the GEMM's epilogue); with x None the product alone.
    a: [T, K] bf16 (rows may be strided), w: [N, K] bf16, x: [T, N] bf16,
    gate_res: [B, N] fp32. out may be x (in place)."""
    import torch
    T, K = a.shape
    N = w.shape[0]
    assert w.shape == (N, K) and w.is_contiguous()
    if out is None:
        out = torch.empty((T, N), dtype=a.dtype, device=a.device)
    B = 0 if cu_seqlens is None else cu_seqlens.shape[0] - 1
    x_stride = 0 if x is None else _token_stride(x, 2)
    _check("pqk_linear_gated_residual", lib().pqk_linear_gated_residual(
        _ptr(a), _token_stride(a, 2), _ptr(w), _ptr(x), x_stride, _ptr(gate_res), _ptr(cu_seqlens), B, _ptr(out),
        _token_stride(out, 2), T, K, N, _stream(stream)))
    return out


def linear_swiglu(a, w1, *, act=None, stream=None):
    """act = silu(a @ w1[:F].T) * (a @ w1[F:].T) on the tensor cores (SwiGLU
    in the GEMM's epilogue). a: [T, K] bf16, w1: [2F, K] bf16."""
    import torch
    T, K = a.shape
    F = w1.shape[0] // 2
    assert w1.shape == (2 * F, K) and w1.is_contiguous()
    if act is None:
        act = torch.empty((T, F), dtype=a.dtype, device=a.device)
    _check("pqk_linear_swiglu", lib().pqk_linear_swiglu(
        _ptr(a), _token_stride(a, 2), _ptr(w1), _ptr(act), _token_stride(act, 2), T, K, F, _stream(stream)))
    return act


def get_device_status(stream=None) -> int:
    return int(lib().pqk_get_device_status(_stream(stream)))


def set_wait_timeout_ns(ns: int) -> None:
    lib().pqk_set_wait_timeout_ns(int(ns))


def set_attn_cta_pairs(enable: bool) -> None:
    """The bf16, head_dim 128 attention on CTA pairs (bit-identical results)."""
    lib().pqk_set_attn_cta_pairs(1 if enable else 0)


def selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check("pqk_selftest_wait_timeout", lib().pqk_selftest_wait_timeout(int(timeout_ns), _stream(stream)))


def version() -> str:
    return lib().pqk_version().decode()
