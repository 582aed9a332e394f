"""The FMA-pipe 2^x used by part of the attention softmax (pqk::ex2_fma in
csrc/sm100_ptx.cuh): its coefficients are the ones the committed fit
(csrc/fit_exp2_poly.py) produces, and a float32 evaluation of the same steps
stays within the fit's relative error bound over the softmax's input range
[-126, 8] (CPU only; the GPU parity tests cover the kernel itself)."""

import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "packed_attention_qk_b200", "csrc", "sm100_ptx.cuh")
FIT = os.path.join(ROOT, "packed_attention_qk_b200", "csrc", "fit_exp2_poly.py")


def header_coefficients():
    body = open(HDR).read().split("float ex2_fma(float x)")[1].split("}")[0]
    # p = fmaf(f, c3, c2); p = fmaf(p, f, c1); p = fmaf(p, f, 1.0f)
    c3, c2 = (float(v) for v in re.search(r"fmaf\(f, ([0-9.]+)f, ([0-9.]+)f\)", body).groups())
    c1, one = (float(v) for v in re.findall(r"fmaf\(p, f, ([0-9.]+)f\)", body))
    assert one == 1.0
    return c1, c2, c3


def test_coefficients_match_the_fit():
    out = subprocess.run([sys.executable, FIT], capture_output=True, text=True, check=True).stdout
    fitted = [float(v) for v in re.search(r"\(c1, c2, c3\): \[([^\]]+)\]", out).group(1).split(",")]
    np.testing.assert_array_equal(np.float32(fitted), np.float32(header_coefficients()))


def ex2_fma_f32(x):
    c1, c2, c3 = (np.float32(c) for c in header_coefficients())
    x = np.maximum(np.float32(x), np.float32(-126.0))
    M = np.float32(12582912.0)
    t = (x + M).astype(np.float32)
    n = (t - M).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), np.arange(-126, 9)]).astype(np.float32)
    got = ex2_fma_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    ok = x >= -125.0   # the lowest binade lands in denormals, where only the magnitude matters
    assert np.max(np.abs(got[ok] / ref[ok] - 1.0)) <= 1.1e-4
    assert np.all(got[~ok] < 2.4e-38) and np.all(got >= 0)
    # integers are exact
    ints = np.arange(-125, 9).astype(np.float32)
    np.testing.assert_array_equal(ex2_fma_f32(ints), np.exp2(ints.astype(np.float64)).astype(np.float32))


def test_masked_scores_are_negligible():
    assert ex2_fma_f32(np.array([-np.inf], np.float32))[0] < 2.4e-38
