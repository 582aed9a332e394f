"""The C-ABI library loads, exports every entry point include/pqk.h declares,
and rejects bad arguments on the host before touching a GPU (CPU only: no
compute call is made; every case below returns before any CUDA call)."""

import os
import re
import subprocess

import pytest

from packed_attention_qk_b200 import build as pqk_build
from packed_attention_qk_b200 import pqk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pqk.h")

ERR_INVALID, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_WORKSPACE = -1, -2, -3, -5
A = 0x10000  # a 16-byte aligned fake device address; never dereferenced on the host
U = 0x10004  # misaligned


@pytest.fixture(scope="module")
def L():
    pqk_build.build()
    return pqk.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"PQK_API\s+[\w\s\*]+?\b(pqk_\w+)\s*\(", text)))


def test_header_declarations_match_binding_list():
    assert declared_functions() == sorted(pqk.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", pqk.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)
    # nothing but the C ABI is exported
    assert {n for n in exported if n.startswith("pqk_")} == set(declared_functions())


def test_library_has_no_libcuda_or_oracle_dependency(L):
    out = subprocess.run(["ldd", pqk.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "oracle" not in out


def test_status_strings_and_version(L):
    assert pqk.status_string(0) == "ok"
    for code in range(-1, -8, -1):
        assert pqk.status_string(code) != "unknown status"
    assert pqk.status_string(-99) == "unknown status"
    assert re.fullmatch(r"\d+\.\d+\.\d+", pqk.version())


def test_workspace_size(L):
    assert L.pqk_varlen_attn_workspace_size(0) == 0
    a, b = L.pqk_varlen_attn_workspace_size(1), L.pqk_varlen_attn_workspace_size(4096)
    assert a > 0 and b > a and a % 256 == 0 and b % 256 == 0
    assert b >= 4 * (2 + 4097 + 2 * 4096)


def qk(L, **kw):
    a = dict(q_in=A, k_in=A, q_out=A, k_out=A, qs=1024, ks=1024, wq=A, wk=A, pos=A, T=16, H=8, D=128, eps=1e-6,
             base=10000.0, style=0)
    a.update(kw)
    qos, kos = a.get("qos", a["qs"]), a.get("kos", a["ks"])
    return L.pqk_qk_norm_rope(a["q_in"], a["k_in"], a["q_out"], a["k_out"], a["qs"], a["ks"], qos, kos, a["wq"],
                              a["wk"], a["pos"], a["T"], a["H"], a["D"], a["eps"], a["base"], a["style"], None)


def test_qk_norm_rope_output_strides(L):
    assert qk(L, qos=1000) == ERR_INVALID             # output stride below H*D
    assert qk(L, qos=1028, q_out=A + 4096) == ERR_MISALIGNED
    assert qk(L, kos=2048) == ERR_INVALID             # in place (k_out == k_in) needs the same stride
    assert qk(L, T=0, qos=3072, kos=3072, q_out=A + 8192, k_out=A + 16384) == 0


def test_qk_norm_rope_e4m3_host_errors(L):
    def call(**kw):
        a = dict(q=A, k=A, q8=A, k8=A, qs=1024, ks=1024, wq=A, wk=A, pos=A, T=16, H=8, D=128, deq=A)
        a.update(kw)
        return L.pqk_qk_norm_rope_e4m3(a["q"], a["k"], a["q8"], a["k8"], a["qs"], a["ks"], a["wq"], a["wk"], a["pos"],
                                       a["T"], a["H"], a["D"], 1e-6, 10000.0, 0, a["deq"], None)
    assert call(D=96) == ERR_UNSUPPORTED
    assert call(qs=1000) == ERR_INVALID
    assert call(deq=None) == ERR_INVALID
    assert call(q8=A + 8) == ERR_MISALIGNED
    assert call(deq=A + 2) == ERR_MISALIGNED
    assert call(T=0, q=None) == 0


def test_qk_norm_rope_host_errors(L):
    assert qk(L, D=96) == ERR_UNSUPPORTED
    assert qk(L, D=256) == ERR_UNSUPPORTED
    assert qk(L, H=0) == ERR_INVALID
    assert qk(L, T=-1) == ERR_INVALID
    assert qk(L, eps=0.0) == ERR_INVALID
    assert qk(L, base=-1.0) == ERR_INVALID
    assert qk(L, style=2) == ERR_INVALID
    assert qk(L, qs=1000) == ERR_INVALID           # < H*D
    assert qk(L, q_in=None) == ERR_INVALID
    assert qk(L, pos=None) == ERR_INVALID
    assert qk(L, k_out=U) == ERR_MISALIGNED
    assert qk(L, wq=U) == ERR_MISALIGNED
    assert qk(L, qs=1028) == ERR_MISALIGNED        # not a multiple of 8 elements
    assert qk(L, T=0, q_in=None) == 0              # empty: nothing to do


def qk3(L, **kw):
    a = dict(q_in=A, k_in=A, q_out=A, k_out=A, qs=1024, ks=1024, wq=A, wk=A, pos=A, st=16, sh=24, sw=24, T=16, H=8,
             D=128, eps=1e-6, base=10000.0, style=0)
    a.update(kw)
    return L.pqk_qk_norm_rope_3axis(a["q_in"], a["k_in"], a["q_out"], a["k_out"], a["qs"], a["ks"], a["wq"],
                                    a["wk"], a["pos"], a["st"], a["sh"], a["sw"], a["T"], a["H"], a["D"], a["eps"],
                                    a["base"], a["style"], None)


def test_qk_norm_rope_3axis_host_errors(L):
    assert qk3(L, sw=23) == ERR_INVALID            # sections must cover D/2 pairs
    assert qk3(L, st=-1, sh=41) == ERR_INVALID
    assert qk3(L, D=64) == ERR_INVALID             # 16 + 24 + 24 != 32
    assert qk3(L, D=96, st=16, sh=16, sw=16) == ERR_UNSUPPORTED
    assert qk3(L, pos=None) == ERR_INVALID
    assert qk3(L, q_out=U) == ERR_MISALIGNED
    assert qk3(L, T=0, q_in=None) == 0


def attn(L, **kw):
    a = dict(q=A, k=A, v=A, o=A, lse=None, qs=1024, ks=1024, vs=1024, os_=1024, cu=A, B=2, T=512, H=8, D=128,
             scale=0.088, ws=A, wsb=4096)
    a.update(kw)
    return L.pqk_varlen_attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["qs"], a["ks"], a["vs"], a["os_"],
                                 a["cu"], a["B"], a["T"], a["H"], a["D"], a["scale"], a["ws"], a["wsb"], None)


def test_varlen_attn_host_errors(L):
    assert attn(L, D=96) == ERR_UNSUPPORTED
    assert attn(L, B=0) == ERR_INVALID
    assert attn(L, H=0) == ERR_INVALID
    assert attn(L, scale=0.0) == ERR_INVALID
    assert attn(L, scale=float("inf")) == ERR_INVALID
    assert attn(L, vs=512) == ERR_INVALID
    assert attn(L, cu=None) == ERR_INVALID
    assert attn(L, o=None) == ERR_INVALID
    assert attn(L, v=U) == ERR_MISALIGNED
    assert attn(L, lse=U) == ERR_MISALIGNED
    assert attn(L, os_=1032 + 4) == ERR_MISALIGNED
    assert attn(L, ws=None) == ERR_WORKSPACE
    assert attn(L, wsb=8) == ERR_WORKSPACE
    assert attn(L, ws=U) == ERR_MISALIGNED
    assert attn(L, T=0, q=None) == 0


def mod(L, **kw):
    a = dict(x=A, br=None, xo=None, h=A, shift=A, scale=A, gr=None, cu=A, B=1, T=8, C=256, nt=0, eps=1e-6,
             gate=A, up=A, gus=512, act=A, F=512)
    a.update(kw)
    return L.pqk_modulate_swiglu(a["x"], a["br"], a["xo"], a["h"], a["shift"], a["scale"], a["gr"], a["cu"], a["B"],
                                 a["T"], a["C"], a["nt"], a["eps"], a["gate"], a["up"], a["gus"], a["act"], a["F"],
                                 None)


def test_attention_rejects_more_work_tiles_than_32_bits_count(L):
    # (ceil(T/256) + B) * H above 2^31 - 2^20: refused on the host for every attention entry
    T, H = 2 ** 31 - 600, 4096
    assert L.pqk_varlen_attn_fwd(A, A, A, A, None, H * 128, H * 128, H * 128, H * 128, A, 1, T, H, 128, 0.1, A,
                                 4096, None) == ERR_INVALID
    assert L.pqk_varlen_attn_fwd_skip(A, A, A, A, None, H * 128, H * 128, H * 128, H * 128, A, 1, T, H, 128, 0.1,
                                      8.0, None, A, 4096, None) == ERR_INVALID
    assert L.pqk_varlen_attn_fwd_fp8qk(A, A, A, A, A, None, H * 128, H * 128, A, 1, T, H, 128, 0.1,
                                       float("inf"), None, A, 4096, None) == ERR_INVALID
    assert L.pqk_varlen_attn_fwd_fp8(A, A, A, A, A, None, H * 128, A, 1, T, H, 128, 0.1, float("inf"), None, A, 4096,
                                     None) == ERR_INVALID
    # (the no-allocation entry looks up its device array first and then forwards to pqk_varlen_attn_fwd, so the
    # same check applies to it on a GPU; without one it stops at the lookup)


def test_modulate_swiglu_host_errors(L):
    assert mod(L, C=250) == ERR_INVALID
    assert mod(L, C=16392) == ERR_INVALID
    assert mod(L, nt=3) == ERR_INVALID
    assert mod(L, eps=0.0) == ERR_INVALID
    assert mod(L, B=0) == ERR_INVALID
    assert mod(L, br=A, gr=None) == ERR_INVALID     # branch needs its gate
    assert mod(L, up=None) == ERR_INVALID           # gate without up
    assert mod(L, F=500, gus=500) == ERR_INVALID
    assert mod(L, gus=256) == ERR_INVALID           # stride < F
    assert mod(L, act=None) == ERR_INVALID
    assert mod(L, x=U) == ERR_MISALIGNED
    assert mod(L, gate=U) == ERR_MISALIGNED
    assert mod(L, gus=1028) == ERR_MISALIGNED
    assert mod(L, T=0, x=None) == 0


def test_selftest_rejects_bad_timeout(L):
    assert L.pqk_selftest_wait_timeout(0, None) == ERR_INVALID
    assert L.pqk_selftest_wait_timeout(20_000_000_000, None) == ERR_INVALID


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="libpqk.so not found"):
        pqk.lib(str(tmp_path / "libpqk.so"))


def attn_skip(L, **kw):
    a = dict(q=A, k=A, v=A, o=A, lse=None, qs=1024, ks=1024, vs=1024, os_=1024, cu=A, B=2, T=512, H=8, D=128,
             scale=0.088, tau=8.0, counts=None, ws=A, wsb=4096)
    a.update(kw)
    return L.pqk_varlen_attn_fwd_skip(a["q"], a["k"], a["v"], a["o"], a["lse"], a["qs"], a["ks"], a["vs"], a["os_"],
                                      a["cu"], a["B"], a["T"], a["H"], a["D"], a["scale"], a["tau"], a["counts"],
                                      a["ws"], a["wsb"], None)


def test_varlen_attn_skip_host_errors(L):
    assert attn_skip(L, tau=-1.0) == ERR_INVALID
    assert attn_skip(L, tau=float("nan")) == ERR_INVALID
    assert attn_skip(L, D=96) == ERR_UNSUPPORTED
    assert attn_skip(L, scale=0.0) == ERR_INVALID
    assert attn_skip(L, counts=A + 4) == ERR_MISALIGNED
    assert attn_skip(L, q=U) == ERR_MISALIGNED
    assert attn_skip(L, ws=None) == ERR_WORKSPACE
    assert attn_skip(L, T=0, q=None) == 0
    assert attn_skip(L, T=0, q=None, tau=float("inf")) == 0


def test_quantize_qk_e4m3_host_errors(L):
    def call(**kw):
        a = dict(q=A, k=A, qs=1024, ks=1024, T=16, H=8, D=128, q8=A, k8=A, sc=A)
        a.update(kw)
        return L.pqk_quantize_qk_e4m3(a["q"], a["k"], a["qs"], a["ks"], a["T"], a["H"], a["D"], a["q8"], a["k8"],
                                      a["sc"], None)
    assert call(D=96) == ERR_UNSUPPORTED
    assert call(H=0) == ERR_INVALID
    assert call(H=5000, qs=5000 * 128, ks=5000 * 128) == ERR_INVALID
    assert call(qs=1000) == ERR_INVALID
    assert call(sc=None) == ERR_INVALID
    assert call(q8=U) == ERR_MISALIGNED
    assert call(sc=U) == ERR_MISALIGNED
    assert call(ks=1028) == ERR_MISALIGNED


def test_varlen_attn_fp8qk_host_errors(L):
    def call(**kw):
        a = dict(q8=A, k8=A, v=A, deq=A, o=A, lse=None, vs=1024, os_=1024, cu=A, B=2, T=512, H=8, D=128,
                 scale=0.088, tau=float("inf"), counts=None, ws=A, wsb=4096)
        a.update(kw)
        return L.pqk_varlen_attn_fwd_fp8qk(a["q8"], a["k8"], a["v"], a["deq"], a["o"], a["lse"], a["vs"], a["os_"],
                                           a["cu"], a["B"], a["T"], a["H"], a["D"], a["scale"], a["tau"],
                                           a["counts"], a["ws"], a["wsb"], None)
    assert call(D=64, vs=512, os_=512) == ERR_UNSUPPORTED
    assert call(deq=None) == ERR_INVALID
    assert call(B=0) == ERR_INVALID
    assert call(vs=512) == ERR_INVALID
    assert call(k8=U) == ERR_MISALIGNED
    assert call(deq=A + 2) == ERR_MISALIGNED
    assert call(ws=None) == ERR_WORKSPACE
    assert call(tau=-1.0) == ERR_INVALID
    assert call(tau=float("nan")) == ERR_INVALID
    assert call(counts=A + 4) == ERR_MISALIGNED
    assert call(T=0, q8=None) == 0


def test_quantize_e4m3_and_fp8_attention_host_errors(L):
    assert L.pqk_quantize_e4m3(A, 1024, 16, 8, 96, A, A, None) == ERR_UNSUPPORTED
    assert L.pqk_quantize_e4m3(A, 1000, 16, 8, 128, A, A, None) == ERR_INVALID
    assert L.pqk_quantize_e4m3(A, 1024, 16, 8, 128, U, A, None) == ERR_MISALIGNED
    assert L.pqk_quantize_e4m3(A, 1024, 16, 8, 128, A, None, None) == ERR_INVALID

    def call(**kw):
        a = dict(q8=A, k8=A, v8=A, deq=A, o=A, lse=None, os_=1024, cu=A, B=2, T=512, H=8, D=128, scale=0.088,
                 tau=float("inf"), counts=None, ws=A, wsb=4096)
        a.update(kw)
        return L.pqk_varlen_attn_fwd_fp8(a["q8"], a["k8"], a["v8"], a["deq"], a["o"], a["lse"], a["os_"], a["cu"],
                                         a["B"], a["T"], a["H"], a["D"], a["scale"], a["tau"], a["counts"], a["ws"],
                                         a["wsb"], None)
    assert call(D=64, os_=512) == ERR_UNSUPPORTED
    assert call(v8=None) == ERR_INVALID
    assert call(v8=U) == ERR_MISALIGNED
    assert call(os_=512) == ERR_INVALID
    assert call(ws=None) == ERR_WORKSPACE
    assert call(tau=-1.0) == ERR_INVALID
    assert call(tau=float("nan")) == ERR_INVALID
    assert call(tau=8.0, counts=A + 4) == ERR_MISALIGNED
    assert call(T=0, q8=None) == 0


def lin(L, **kw):
    a = dict(a=A, a_stride=256, w=A, x=A, x_stride=512, gr=A, cu=A, B=2, out=A, out_stride=512, T=300, K=256, N=512)
    a.update(kw)
    return L.pqk_linear_gated_residual(a["a"], a["a_stride"], a["w"], a["x"], a["x_stride"], a["gr"], a["cu"], a["B"],
                                       a["out"], a["out_stride"], a["T"], a["K"], a["N"], None)


def test_linear_gated_residual_host_errors(L):
    assert lin(L, K=12) == ERR_INVALID                       # K not a multiple of 8
    assert lin(L, N=4) == ERR_INVALID
    assert lin(L, T=-1) == ERR_INVALID
    assert lin(L, T=2 ** 31) == ERR_INVALID                  # token coordinates are int32
    assert lin(L, a_stride=128) == ERR_INVALID               # stride below K
    assert lin(L, out_stride=256) == ERR_INVALID
    assert lin(L, gr=None) == ERR_INVALID                    # x without its gate
    assert lin(L, x=None) == ERR_INVALID                     # gate without x
    assert lin(L, cu=None) == ERR_INVALID
    assert lin(L, B=0) == ERR_INVALID
    assert lin(L, x_stride=256) == ERR_INVALID
    assert lin(L, T=0) == 0                                   # nothing to do, nothing enqueued
    assert lin(L, a=None) == ERR_INVALID
    assert lin(L, w=U) == ERR_MISALIGNED
    assert lin(L, out=U) == ERR_MISALIGNED
    assert lin(L, a_stride=260) == ERR_MISALIGNED             # rows not 16-byte aligned
    assert lin(L, x=None, gr=None, cu=None, B=0, x_stride=0, a=U) == ERR_MISALIGNED   # the product alone
    # more output tiles than 32-bit tile indices can count
    assert lin(L, T=2 ** 31 - 300, N=2 ** 30, x_stride=2 ** 30, out_stride=2 ** 30) == ERR_INVALID


def test_linear_swiglu_host_errors(L):
    f = lambda **kw: L.pqk_linear_swiglu(kw.get("a", A), kw.get("a_stride", 256), kw.get("w1", A), kw.get("act", A),
                                         kw.get("act_stride", 512), kw.get("T", 300), kw.get("K", 256),
                                         kw.get("F", 512), None)
    assert f(K=20) == ERR_INVALID
    assert f(F=4) == ERR_INVALID
    assert f(act_stride=500) == ERR_INVALID
    assert f(T=0) == 0
    assert f(w1=None) == ERR_INVALID
    assert f(act=U) == ERR_MISALIGNED
    assert f(act_stride=516) == ERR_MISALIGNED
    assert f(T=2 ** 31 - 300, F=2 ** 30, act_stride=2 ** 30) == ERR_INVALID
