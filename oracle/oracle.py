"""Python access to the float64 CPU oracle (``pqk_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
bench's CPU-baseline leg, never by the library. It shares no code with the
CUDA path. Inputs are numpy arrays (bfloat16 as uint16 bit patterns, or
float64); outputs are float64.
"""

from __future__ import annotations

import ctypes as C
import math
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pqk_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

ROPE_INTERLEAVED, ROPE_HALF = 0, 1
NORM_RMS, NORM_LAYER, NORM_NONE = 0, 1, 2
_IN_BF16, _IN_F64 = 0, 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no fast-math)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


def load(path: str):
    """Load an oracle build from ``path`` and declare its signatures."""
    L = C.CDLL(path)
    vp, i32p, f32p, f64p = C.c_void_p, C.POINTER(C.c_int32), C.POINTER(C.c_float), C.POINTER(C.c_double)
    L.oracle_qk_norm_rope.argtypes = [vp, C.c_int, C.c_int64, vp, C.c_int, i32p, C.c_int64, C.c_int,
                                      C.c_int, C.c_double, C.c_double, C.c_int, i32p, C.c_int64, f64p]
    L.oracle_varlen_attn.argtypes = [vp, vp, vp, C.c_int, C.c_int64, i32p, C.c_int, C.c_int64, C.c_int,
                                     C.c_int, C.c_double, i32p, C.c_int64, f64p, f64p]
    L.oracle_modulate_swiglu.argtypes = [vp, vp, C.c_int, f32p, f32p, f32p, i32p, C.c_int, C.c_int64,
                                         C.c_int, C.c_int, C.c_double, vp, vp, C.c_int64, C.c_int, i32p,
                                         C.c_int64, f64p, f64p, f64p]
    L.oracle_qk_norm_rope_3axis.argtypes = [vp, C.c_int, C.c_int64, vp, C.c_int, i32p, i32p, C.c_int64, C.c_int,
                                            C.c_int, C.c_double, C.c_double, C.c_int, i32p, C.c_int64, f64p]
    L.oracle_qk_fullc_norm_rope.argtypes = [vp, C.c_int, C.c_int64, vp, C.c_int, i32p, C.c_int64, C.c_int, C.c_int,
                                            C.c_double, C.c_double, C.c_int, i32p, C.c_int64, f64p]
    L.oracle_varlen_attn_skip.argtypes = [vp, vp, vp, C.c_int, C.c_int64, i32p, C.c_int, C.c_int64, C.c_int,
                                          C.c_int, C.c_double, C.c_double, C.c_int, C.c_int, C.c_int, i32p,
                                          C.c_int64, f64p, f64p, C.POINTER(C.c_int64)]
    u8p = C.POINTER(C.c_uint8)
    L.oracle_quantize_e4m3.argtypes = [vp, C.c_int, C.c_int64, C.c_int64, C.c_int, C.c_int, u8p, f32p]
    L.oracle_varlen_attn_fp8qk.argtypes = [vp, vp, vp, C.c_int, C.c_int64, i32p, C.c_int, C.c_int64, C.c_int,
                                           C.c_int, C.c_double, C.c_double, C.c_int, C.c_int, C.c_int, i32p,
                                           C.c_int64, f64p, f64p, C.POINTER(C.c_int64), u8p, u8p, f32p]
    skip_args = [C.c_double, C.c_int, C.c_int, C.c_int]  # tau, query rows, keys, tile rows
    L.oracle_varlen_attn_fp8.argtypes = [vp, vp, vp, C.c_int, C.c_int64, i32p, C.c_int, C.c_int64, C.c_int,
                                         C.c_int, C.c_double, *skip_args, i32p, C.c_int64, f64p, f64p,
                                         C.POINTER(C.c_int64), f32p]
    L.oracle_varlen_attn_fp8_online.argtypes = [vp, vp, vp, C.c_int, C.c_int64, i32p, C.c_int, C.c_int64, C.c_int,
                                                C.c_int, C.c_double, C.c_int, C.c_double, *skip_args, i32p,
                                                C.c_int64, f64p, f64p, C.POINTER(C.c_int64), f32p]
    L.oracle_linear_gated_residual.argtypes = [vp, C.c_int64, vp, vp, C.c_int, f32p, i32p, C.c_int, C.c_int64,
                                               C.c_int, C.c_int, i32p, C.c_int64, f64p]
    L.oracle_linear_swiglu.argtypes = [vp, C.c_int64, vp, C.c_int, C.c_int64, C.c_int, C.c_int, i32p, C.c_int64,
                                       f64p]
    L.oracle_qk_norm_rope_e4m3.argtypes = [vp, C.c_int, C.c_int64, vp, C.c_int, i32p, C.c_int64, C.c_int, C.c_int,
                                           C.c_double, C.c_double, C.c_int, i32p, C.c_int64, u8p, f32p]
    L.oracle_e4m3_codes.argtypes = [f32p, C.c_int64, u8p]
    L.oracle_e4m3_codes.restype = None
    for f in (L.oracle_qk_norm_rope, L.oracle_qk_norm_rope_e4m3, L.oracle_qk_norm_rope_3axis, L.oracle_qk_fullc_norm_rope, L.oracle_varlen_attn,
              L.oracle_varlen_attn_skip, L.oracle_quantize_e4m3, L.oracle_varlen_attn_fp8qk, L.oracle_varlen_attn_fp8,
              L.oracle_varlen_attn_fp8_online, L.oracle_modulate_swiglu, L.oracle_linear_gated_residual, L.oracle_linear_swiglu):
        f.restype = C.c_int
    L.oracle_num_threads.restype = C.c_int
    L.oracle_set_num_threads.argtypes = [C.c_int]
    L.oracle_set_num_threads.restype = None
    return L


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load(LIB)
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of later oracle calls (timing only; results do not depend on it)."""
    lib().oracle_set_num_threads(int(n))


def _kind(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return _IN_BF16
    if a.dtype == np.float64:
        return _IN_F64
    raise TypeError(f"oracle inputs are bf16 bits (uint16) or float64, got {a.dtype}")


def _ptr(a, ctype=None):
    if a is None:
        return None
    if ctype is None:
        return a.ctypes.data_as(C.c_void_p)
    return a.ctypes.data_as(C.POINTER(ctype))


def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int32)
    return r, int(r.shape[0])


def qk_norm_rope(x: np.ndarray, w: np.ndarray, pos: np.ndarray, eps: float, base: float,
                 style: int = ROPE_INTERLEAVED, rows=None) -> np.ndarray:
    """x: [T, H, D] (a strided view over a wider token row is allowed)."""
    T, H, D = x.shape
    stride_t = x.strides[0] // x.itemsize
    assert x.strides[2] == x.itemsize and x.strides[1] == D * x.itemsize
    # a strided token view is passed by its first element; stride_t covers
    # the gap between tokens
    w = np.ascontiguousarray(w)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    r, n = _rows(rows)
    y = np.empty((n if r is not None else T, H, D), np.float64)
    rc = lib().oracle_qk_norm_rope(_ptr(x), _kind(x), stride_t, _ptr(w), _kind(w), _ptr(pos, C.c_int32),
                                   T, H, D, eps, base, style, _ptr(r, C.c_int32), n, _ptr(y, C.c_double))
    if rc:
        raise ValueError("oracle_qk_norm_rope: invalid arguments")
    return y


def qk_norm_rope_e4m3(x: np.ndarray, w: np.ndarray, pos: np.ndarray, eps: float, base: float,
                      style: int = ROPE_INTERLEAVED, rows=None):
    """RMSNorm + RoPE, then e4m3 codes with the per-tensor scale of the bound
    sqrt(D) * max|w| (oracle_qk_norm_rope_e4m3). Returns (codes uint8
    [nrows, H, D], deq float32)."""
    T, H, D = x.shape
    stride_t = x.strides[0] // x.itemsize
    assert x.strides[2] == x.itemsize and x.strides[1] == D * x.itemsize
    w = np.ascontiguousarray(w)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    r, n = _rows(rows)
    codes = np.empty((n if r is not None else T, H, D), np.uint8)
    deq = np.empty(1, np.float32)
    rc = lib().oracle_qk_norm_rope_e4m3(_ptr(x), _kind(x), stride_t, _ptr(w), _kind(w), _ptr(pos, C.c_int32), T, H, D,
                                        eps, base, style, _ptr(r, C.c_int32), n, _ptr(codes, C.c_uint8),
                                        _ptr(deq, C.c_float))
    if rc:
        raise ValueError("oracle_qk_norm_rope_e4m3: invalid arguments")
    return codes, deq[0]


def qk_norm_rope_3axis(x: np.ndarray, w: np.ndarray, pos3: np.ndarray, sections, eps: float, base: float,
                       style: int = ROPE_INTERLEAVED, rows=None) -> np.ndarray:
    """x: [T, H, D]; pos3: [T, 3] (t, h, w) ids; sections: pairs per axis."""
    T, H, D = x.shape
    stride_t = x.strides[0] // x.itemsize
    assert x.strides[2] == x.itemsize and x.strides[1] == D * x.itemsize
    w = np.ascontiguousarray(w)
    pos3 = np.ascontiguousarray(pos3, dtype=np.int32)
    assert pos3.shape == (T, 3)
    sec = np.ascontiguousarray(sections, dtype=np.int32)
    r, n = _rows(rows)
    y = np.empty((n if r is not None else T, H, D), np.float64)
    rc = lib().oracle_qk_norm_rope_3axis(_ptr(x), _kind(x), stride_t, _ptr(w), _kind(w), _ptr(pos3, C.c_int32),
                                         _ptr(sec, C.c_int32), T, H, D, eps, base, style, _ptr(r, C.c_int32), n,
                                         _ptr(y, C.c_double))
    if rc:
        raise ValueError("oracle_qk_norm_rope_3axis: invalid arguments")
    return y


def qk_fullc_norm_rope(x: np.ndarray, w: np.ndarray, pos: np.ndarray, eps: float, base: float,
                       style: int = ROPE_INTERLEAVED, rows=None) -> np.ndarray:
    """x: [T, H, D]; w: [H*D]; RMS over all H*D elements of a token."""
    T, H, D = x.shape
    stride_t = x.strides[0] // x.itemsize
    assert x.strides[2] == x.itemsize and x.strides[1] == D * x.itemsize
    w = np.ascontiguousarray(w).reshape(-1)
    assert w.shape[0] == H * D
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    r, n = _rows(rows)
    y = np.empty((n if r is not None else T, H, D), np.float64)
    rc = lib().oracle_qk_fullc_norm_rope(_ptr(x), _kind(x), stride_t, _ptr(w), _kind(w), _ptr(pos, C.c_int32), T, H,
                                         D, eps, base, style, _ptr(r, C.c_int32), n, _ptr(y, C.c_double))
    if rc:
        raise ValueError("oracle_qk_fullc_norm_rope: invalid arguments")
    return y


def varlen_attn(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens: np.ndarray, scale: float,
                rows=None, want_lse: bool = True):
    """q, k, v: [T, H, D] contiguous. Returns (o [nrows, H, D], lse [nrows, H])."""
    T, H, D = q.shape
    assert k.shape == q.shape == v.shape and q.dtype == k.dtype == v.dtype
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    r, n = _rows(rows)
    n = n if r is not None else T
    o = np.empty((n, H, D), np.float64)
    lse = np.empty((n, H), np.float64) if want_lse else None
    rc = lib().oracle_varlen_attn(_ptr(q), _ptr(k), _ptr(v), _kind(q), H * D, _ptr(cu, C.c_int32),
                                  int(cu.shape[0]) - 1, T, H, D, scale, _ptr(r, C.c_int32), n if r is not None else 0,
                                  _ptr(o, C.c_double), _ptr(lse, C.c_double))
    if rc:
        raise ValueError("oracle_varlen_attn: invalid arguments")
    return o, lse


def varlen_attn_skip(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens: np.ndarray, scale: float, tau: float,
                     *, block, tile_rows: int, rows=None, want_lse: bool = True):
    """Attention with key blocks skipped where negligible (oracle_varlen_attn_skip).
    block = (query rows, keys) of a decision block; tile_rows (a multiple of
    the block's rows) groups query blocks for the second count. Returns
    (o [nrows, H, D], lse [nrows, H] or None, counts): counts is (skipped
    query blocks, skipped tiles) over all (block, head, key block) triples
    when rows is None, else None."""
    T, H, D = q.shape
    assert k.shape == q.shape == v.shape and q.dtype == k.dtype == v.dtype
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    qrows, kblock = (int(b) for b in block)
    r, n = _rows(rows)
    n = n if r is not None else T
    o = np.empty((n, H, D), np.float64)
    lse = np.empty((n, H), np.float64) if want_lse else None
    counts = np.zeros(2, np.int64)
    rc = lib().oracle_varlen_attn_skip(_ptr(q), _ptr(k), _ptr(v), _kind(q), H * D, _ptr(cu, C.c_int32),
                                       int(cu.shape[0]) - 1, T, H, D, scale, float(tau), qrows, kblock,
                                       int(tile_rows), _ptr(r, C.c_int32), n if r is not None else 0,
                                       _ptr(o, C.c_double), _ptr(lse, C.c_double), _ptr(counts, C.c_int64))
    if rc:
        raise ValueError("oracle_varlen_attn_skip: invalid arguments")
    return o, lse, (tuple(int(c) for c in counts) if r is None else None)


def e4m3_codes(x: np.ndarray) -> np.ndarray:
    """FP8 e4m3 codes (uint8) of float32 values: nearest, ties to even,
    magnitudes beyond 448 saturating to 448."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().oracle_e4m3_codes(_ptr(x, C.c_float), x.size, _ptr(out, C.c_uint8))
    return out


def quantize_e4m3(x: np.ndarray):
    """Per-head absmax e4m3 quantisation of [T, H, D]: (codes uint8 [T, H, D], deq float32 [H])."""
    T, H, D = x.shape
    x = np.ascontiguousarray(x)
    codes = np.empty((T, H, D), np.uint8)
    deq = np.empty(H, np.float32)
    if lib().oracle_quantize_e4m3(_ptr(x), _kind(x), H * D, T, H, D, _ptr(codes, C.c_uint8), _ptr(deq, C.c_float)):
        raise ValueError("oracle_quantize_e4m3: invalid arguments")
    return codes, deq


def varlen_attn_fp8qk(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens: np.ndarray, scale: float, rows=None,
                      want_lse: bool = True, tau: float = math.inf, skip_block=None, skip_tile_rows=None,
                      counts_out: list | None = None):
    """Attention with Q and K quantised to e4m3 per head (block skipping on
    the quantised scores for a finite tau, with the geometry skip_block =
    (query rows, keys) and skip_tile_rows as in varlen_attn_skip; its counts
    appended to counts_out when given). Returns (o [nrows, H, D], lse
    [nrows, H] or None, q8, k8 [T, H, D] uint8, deq [2H])."""
    T, H, D = q.shape
    assert k.shape == q.shape == v.shape and q.dtype == k.dtype == v.dtype
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    tau, qrows, kblock, tile_rows = _skip_geometry(tau, skip_block, skip_tile_rows)
    r, n = _rows(rows)
    n = n if r is not None else T
    o = np.empty((n, H, D), np.float64)
    lse = np.empty((n, H), np.float64) if want_lse else None
    q8 = np.empty((T, H, D), np.uint8)
    k8 = np.empty((T, H, D), np.uint8)
    deq = np.empty(2 * H, np.float32)
    counts = np.zeros(2, np.int64)
    rc = lib().oracle_varlen_attn_fp8qk(_ptr(q), _ptr(k), _ptr(v), _kind(q), H * D, _ptr(cu, C.c_int32),
                                        int(cu.shape[0]) - 1, T, H, D, scale, tau, qrows, kblock, tile_rows,
                                        _ptr(r, C.c_int32), n if r is not None else 0, _ptr(o, C.c_double),
                                        _ptr(lse, C.c_double), _ptr(counts, C.c_int64), _ptr(q8, C.c_uint8),
                                        _ptr(k8, C.c_uint8), _ptr(deq, C.c_float))
    if rc:
        raise ValueError("oracle_varlen_attn_fp8qk: invalid arguments")
    if counts_out is not None and r is None:
        counts_out.append(tuple(int(c) for c in counts))
    return o, lse, q8, k8, deq


def _skip_geometry(tau, skip_block, skip_tile_rows):
    """(tau, query rows, keys, tile rows) for the C calls; the geometry is
    unused (and not needed) for an infinite tau."""
    if math.isinf(tau) and tau > 0:
        return float(tau), 1, 1, 1
    if skip_block is None or skip_tile_rows is None:
        raise ValueError("a finite tau needs the block geometry (skip_block, skip_tile_rows)")
    qrows, kblock = (int(b) for b in skip_block)
    return float(tau), qrows, kblock, int(skip_tile_rows)


def _fp8_call(fn, name, q, k, v, cu_seqlens, scale, rows, want_lse, extra, skip, counts_out):
    T, H, D = q.shape
    assert k.shape == q.shape == v.shape and q.dtype == k.dtype == v.dtype
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    r, n = _rows(rows)
    n = n if r is not None else T
    o = np.empty((n, H, D), np.float64)
    lse = np.empty((n, H), np.float64) if want_lse else None
    deq = np.empty(3 * H, np.float32)
    counts = np.zeros(2, np.int64)
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _kind(q), H * D, _ptr(cu, C.c_int32), int(cu.shape[0]) - 1, T, H, D, scale,
            *extra, *skip, _ptr(r, C.c_int32), n if r is not None else 0, _ptr(o, C.c_double), _ptr(lse, C.c_double),
            _ptr(counts, C.c_int64), _ptr(deq, C.c_float))
    if rc:
        raise ValueError(f"{name}: invalid arguments")
    if counts_out is not None and not (math.isinf(skip[0]) and skip[0] > 0):
        counts_out.append(tuple(int(c) for c in counts))
    return o, lse, deq


def varlen_attn_fp8(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens: np.ndarray, scale: float, rows=None,
                    want_lse: bool = True, tau: float = math.inf, skip_block=None, skip_tile_rows=None,
                    counts_out: list | None = None):
    """Attention with Q, K, V and P in FP8 e4m3, P rounded against each row's
    exact maximum (oracle_varlen_attn_fp8); with a finite tau, key blocks are
    skipped by the rule of varlen_attn_skip on the dequantised Q, K (geometry
    skip_block = (query rows, keys), skip_tile_rows; the counts of all T rows
    appended to counts_out). Returns (o [nrows, H, D], lse [nrows, H] or
    None, deq [3H])."""
    return _fp8_call(lib().oracle_varlen_attn_fp8, "oracle_varlen_attn_fp8", q, k, v, cu_seqlens, scale, rows,
                     want_lse, (), _skip_geometry(tau, skip_block, skip_tile_rows), counts_out)


def varlen_attn_fp8_online(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens: np.ndarray, scale: float, *,
                           kblock: int, threshold: float, rows=None, want_lse: bool = True, tau: float = math.inf,
                           skip_block=None, skip_tile_rows=None, counts_out: list | None = None):
    """The same FP8 attention in the rounding order of an online softmax over
    blocks of kblock keys whose running maximum moves only past threshold
    (log2 units): a streaming implementation's schedule, not the definition
    (oracle_varlen_attn_fp8_online). Block skipping as in varlen_attn_fp8.
    Returns (o, lse or None, deq [3H])."""
    return _fp8_call(lib().oracle_varlen_attn_fp8_online, "oracle_varlen_attn_fp8_online", q, k, v, cu_seqlens,
                     scale, rows, want_lse, (int(kblock), float(threshold)),
                     _skip_geometry(tau, skip_block, skip_tile_rows), counts_out)


def modulate_swiglu(x: np.ndarray, shift: np.ndarray, scale: np.ndarray, gate_res: np.ndarray,
                    cu_seqlens: np.ndarray, norm_type: int = NORM_RMS, eps: float = 1e-6,
                    branch=None, gate=None, up=None, rows=None):
    """Returns (x_out or None, h, act or None), float64."""
    T, Cdim = x.shape
    x = np.ascontiguousarray(x)
    if branch is not None:
        branch = np.ascontiguousarray(branch)
        assert branch.dtype == x.dtype and branch.shape == x.shape
    shift, scale, gate_res = (np.ascontiguousarray(a, dtype=np.float32) for a in (shift, scale, gate_res))
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    F, gu_stride = 0, 0
    if gate is not None:
        assert up is not None and gate.shape == up.shape and gate.dtype == x.dtype
        F = gate.shape[1]
        gate, up = np.ascontiguousarray(gate), np.ascontiguousarray(up)
        gu_stride = F
    r, n = _rows(rows)
    n = n if r is not None else T
    xo = np.empty((n, Cdim), np.float64) if branch is not None else None
    h = np.empty((n, Cdim), np.float64)
    act = np.empty((n, F), np.float64) if gate is not None else None
    rc = lib().oracle_modulate_swiglu(_ptr(x), _ptr(branch), _kind(x), _ptr(shift, C.c_float),
                                      _ptr(scale, C.c_float), _ptr(gate_res, C.c_float), _ptr(cu, C.c_int32),
                                      int(cu.shape[0]) - 1, T, Cdim, norm_type, eps, _ptr(gate), _ptr(up),
                                      gu_stride, F, _ptr(r, C.c_int32), n if r is not None else 0,
                                      _ptr(xo, C.c_double), _ptr(h, C.c_double), _ptr(act, C.c_double))
    if rc:
        raise ValueError("oracle_modulate_swiglu: invalid arguments")
    return xo, h, act


def _token_rows(a: np.ndarray):
    """A [T, K] array whose rows may be a strided view: (array, row stride)."""
    assert a.ndim == 2 and a.strides[1] == a.itemsize
    return a, a.strides[0] // a.itemsize


def linear_gated_residual(a: np.ndarray, w: np.ndarray, x=None, gate_res=None, cu_seqlens=None, rows=None):
    """x + gate_res[request] * (a @ w.T) per token (a: [T, K], w: [N, K],
    x: [T, N]); with x None the product alone. float64 [rows, N]."""
    a, a_stride = _token_rows(a)
    T, K = a.shape
    w = np.ascontiguousarray(w)
    N = w.shape[0]
    assert w.shape == (N, K) and w.dtype == a.dtype
    B, cu, g = 0, None, None
    if x is not None:
        x = np.ascontiguousarray(x)
        assert x.shape == (T, N) and x.dtype == a.dtype
        g = np.ascontiguousarray(gate_res, dtype=np.float32)
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
        B = int(cu.shape[0]) - 1
        assert g.shape == (B, N)
    r, n = _rows(rows)
    out = np.empty((n if r is not None else T, N), np.float64)
    rc = lib().oracle_linear_gated_residual(_ptr(a), a_stride, _ptr(w), _ptr(x), _kind(a), _ptr(g, C.c_float),
                                            _ptr(cu, C.c_int32), B, T, K, N, _ptr(r, C.c_int32), n, _ptr(out, C.c_double))
    if rc:
        raise ValueError("oracle_linear_gated_residual: invalid arguments")
    return out


def linear_swiglu(a: np.ndarray, w1: np.ndarray, rows=None):
    """silu(a @ w1[:F].T) * (a @ w1[F:].T) per token (a: [T, K], w1: [2F, K]).
    float64 [rows, F]."""
    a, a_stride = _token_rows(a)
    T, K = a.shape
    w1 = np.ascontiguousarray(w1)
    assert w1.ndim == 2 and w1.shape[1] == K and w1.shape[0] % 2 == 0 and w1.dtype == a.dtype
    F = w1.shape[0] // 2
    r, n = _rows(rows)
    act = np.empty((n if r is not None else T, F), np.float64)
    rc = lib().oracle_linear_swiglu(_ptr(a), a_stride, _ptr(w1), _kind(a), T, K, F, _ptr(r, C.c_int32), n,
                                    _ptr(act, C.c_double))
    if rc:
        raise ValueError("oracle_linear_swiglu: invalid arguments")
    return act
