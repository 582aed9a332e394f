"""Failure detection on the GPU without a GPU fault.

Every pipeline wait of the attention and linear-layer kernels is bounded by
the library's timeout (pqk_set_wait_timeout_ns). A wait that runs out
records PQK_ERR_TIMEOUT in the device status word; the block stops issuing
work, waits for its copies and MMAs in flight (with a fixed bound of its
own), frees its tensor memory and exits, and the context stays usable.
Nothing here faults, traps or hangs the GPU: the waits run out either on a
barrier that nothing completes (the self-test kernel) or because the
timeout is set shorter (1 us, the smallest the library accepts) than the
real pipelines' copy and MMA latencies. The host reads the status after a
synchronisation, as the serving pages' video-sync timeout does on its side.
"""

import contextlib
import math
import time

import numpy as np
import pytest

from oracle import oracle
from packed_attention_qk_b200 import pqk
from packed_attention_qk_b200 import workloads as wl
from tests.gpu_utils import (LSE_MAX_ABS, assert_attention, assert_elementwise, bf16_to_f64, max_abs, to_dev,
                             to_dev_bf16, torch_cuda)

pytestmark = pytest.mark.gpu

TIMEOUT = -6


@contextlib.contextmanager
def short_timeout(ns):
    pqk.set_wait_timeout_ns(ns)
    try:
        yield
    finally:
        pqk.set_wait_timeout_ns(0)  # back to the default


def test_bounded_wait_times_out_and_context_survives():
    torch = torch_cuda()
    assert pqk.get_device_status() == 0
    t0 = time.time()
    pqk.selftest_wait_timeout(50_000_000)      # 50 ms
    assert pqk.get_device_status() == TIMEOUT
    assert time.time() - t0 < 10.0
    assert pqk.get_device_status() == 0
    # the context still runs real work correctly
    w = wl.config(1)
    x = wl.attention_inputs(w)
    o, _ = pqk.varlen_attn_fwd(to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), to_dev_bf16(x["v"]),
                               to_dev(x["cu_seqlens"]))
    torch.cuda.synchronize()
    ro, _ = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], w.D ** -0.5)
    assert_attention(bf16_to_f64(o), ro, "after timeout")
    assert pqk.get_device_status() == 0


def _runs_out(call, tries=3):
    """Runs call() under the shortest timeout until a wait runs out (each
    run checked for a clean status or PQK_ERR_TIMEOUT); True if one did."""
    with short_timeout(1000):
        for _ in range(tries):
            call()
            st = pqk.get_device_status()
            assert st in (0, TIMEOUT), f"unexpected status {st}"
            if st == TIMEOUT:
                return True
    return False


def test_attention_pipeline_timeout_is_reported_drained_and_recovered():
    torch = torch_cuda()
    w = wl.custom([4096, 1000, 0, 129], 8, 128, seed=61)
    x = wl.attention_inputs(w)
    T, H, D = w.T, w.H, w.D
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    cu = to_dev(x["cu_seqlens"])
    # outputs inside guard bands: 8 rows before and after O, a wider row, and
    # 32 floats on each side of the LSE
    o_full = torch.full((T + 16, H * D + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    o = o_full[8:8 + T, :H * D].view(T, H, D)
    lse_full = torch.full((H * T + 64,), 7.0, dtype=torch.float32, device="cuda")
    lse = lse_full[32:32 + H * T].view(H, T)
    assert _runs_out(lambda: pqk.varlen_attn_fwd(q, k, v, cu, o=o, lse=lse))
    guard = torch.cat([o_full[:8].flatten(), o_full[8 + T:].flatten(), o_full[8:8 + T, H * D:].flatten()])
    assert bool((guard == 7.0).all()), "written outside O"
    assert bool((lse_full[:32] == 7.0).all()) and bool((lse_full[32 + H * T:] == 7.0).all()), "written outside LSE"
    # the next call with the default timeout is correct
    o2, lse2 = pqk.varlen_attn_fwd(q, k, v, cu, want_lse=True)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    scale = 1.0 / math.sqrt(D)
    rows = wl.sample_rows(w, 64)
    ro, rl = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu_seqlens"], scale, rows=rows)
    assert_attention(bf16_to_f64(o2)[rows], ro, "attention after a timed-out call")
    assert max_abs(lse2.cpu().numpy().astype(np.float64).T[rows], rl) <= LSE_MAX_ABS


def test_linear_pipeline_timeout_is_reported_drained_and_recovered():
    # K = 16,384: each output tile's main loop runs for tens of microseconds,
    # so the epilogue's wait for a finished accumulator outlasts the 1 us bound
    torch = torch_cuda()
    g = np.random.default_rng(71)
    lens, K, N = [1500, 0, 548], 16384, 2048
    T = sum(lens)
    a_bits = wl.f32_to_bf16_bits(g.standard_normal((T, K)).astype(np.float32))
    w_bits = wl.f32_to_bf16_bits((g.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    x_bits = wl.f32_to_bf16_bits(g.standard_normal((T, N)).astype(np.float32))
    gate_res = (0.1 * g.standard_normal((len(lens), N))).astype(np.float32)
    cu_np = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    a, wt, x = to_dev_bf16(a_bits), to_dev_bf16(w_bits), to_dev_bf16(x_bits)
    gr, cu = to_dev(gate_res), to_dev(cu_np)
    out_full = torch.full((T + 16, N + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    out = out_full[8:8 + T, :N]
    assert _runs_out(lambda: pqk.linear_gated_residual(a, wt, x=x, gate_res=gr, cu_seqlens=cu, out=out))
    guard = torch.cat([out_full[:8].flatten(), out_full[8 + T:].flatten(), out_full[8:8 + T, N:].flatten()])
    assert bool((guard == 7.0).all()), "written outside the output"
    y = pqk.linear_gated_residual(a, wt, x=x, gate_res=gr, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert pqk.get_device_status() == 0
    rows = np.array(sorted({0, 1, 255, 256, 1499, 1500, 1501, 2047} | set(g.choice(T, 40, replace=False).tolist())),
                    np.int32)
    ref = oracle.linear_gated_residual(a_bits, w_bits, x_bits, gate_res, cu_np, rows=rows)
    assert_elementwise(bf16_to_f64(y)[rows], ref, "linear layer after a timed-out call")


def test_timeout_setting_is_clamped_not_rejected():
    # any value is accepted; tiny ones are raised to 1 us, which still lets a
    # short attention finish or report a timeout, never anything else
    torch = torch_cuda()
    w = wl.config(1)
    x = wl.attention_inputs(w)
    with short_timeout(1):
        pqk.varlen_attn_fwd(to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), to_dev_bf16(x["v"]), to_dev(x["cu_seqlens"]))
        torch.cuda.synchronize()
        assert pqk.get_device_status() in (0, TIMEOUT)
    assert pqk.get_device_status() == 0
