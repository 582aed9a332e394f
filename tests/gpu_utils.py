"""Helpers of the GPU parity tests: bf16 bit patterns between numpy and
torch, and the error metrics with their bounds.

Tolerances (float64 oracle on the same bf16 inputs):
  * elementwise kernels: unit-scale max error max|g - r| / max(1, |r|) <= 1e-2
    and relative L2 ||g - r|| / ||r|| <= 5e-3. A correctly rounded fp32
    result stored as bf16 is within half an ulp, 2^-9 relative, of r.
  * attention: max |g - r| <= 2e-2 and relative L2 <= 1e-2 (bf16 inputs,
    bf16 probabilities, fp32 accumulation); for peaked inputs, where O is
    close to single V rows of size ~1-4, the unit-scale max error <= 1e-2 as
    well.
"""

import numpy as np
import pytest

ELEM_UNIT_MAX = 1e-2
ELEM_REL_L2 = 5e-3
ATTN_MAX_ABS = 2e-2
ATTN_REL_L2 = 1e-2
LSE_MAX_ABS = 1e-3

# The attention kernel's block-skipping geometry: a decision covers one
# softmax warp's 32 query rows x one K/V tile of 128 keys, and a P x V
# product (the second count) one 128-row query tile.
SKIP_BLOCK = (32, 128)
SKIP_TILE_ROWS = 128


def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def to_dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_to_f64(t) -> np.ndarray:
    from packed_attention_qk_b200.workloads import bf16_bits_to_f64
    return bf16_bits_to_f64(t.contiguous().view(__import__("torch").int16).cpu().numpy().view(np.uint16))


def unit_max(g, r) -> float:
    return float(np.max(np.abs(g - r) / np.maximum(1.0, np.abs(r)))) if r.size else 0.0


def rel_l2(g, r) -> float:
    n = np.linalg.norm(r)
    return float(np.linalg.norm(g - r) / n) if n > 0 else float(np.linalg.norm(g - r))


def max_abs(g, r) -> float:
    return float(np.max(np.abs(g - r))) if r.size else 0.0


def assert_elementwise(g, r, what=""):
    u, l2 = unit_max(g, r), rel_l2(g, r)
    assert u <= ELEM_UNIT_MAX and l2 <= ELEM_REL_L2, f"{what}: unit-scale max {u:.3e}, rel-L2 {l2:.3e}"


def assert_attention(g, r, what="", peaked=False):
    m, l2 = max_abs(g, r), rel_l2(g, r)
    assert m <= ATTN_MAX_ABS and l2 <= ATTN_REL_L2, f"{what}: max-abs {m:.3e}, rel-L2 {l2:.3e}"
    if peaked:
        u = unit_max(g, r)
        assert u <= ELEM_UNIT_MAX, f"{what}: unit-scale max {u:.3e}"
