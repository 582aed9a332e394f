"""The oracle's pins must catch plausible mistakes (CPU only).

Each case plants one mistake in a private copy of the oracle's C source (a
dropped term, a wrong sign, index or exponent, swapped operands), builds it,
points the oracle wrapper at that build and runs every pin of the three
oracle test modules against it. A mutant that no pin rejects means the pins
are too weak. Mistakes are planted only in the oracle, only on the CPU.
"""

import inspect
import itertools
import os
import subprocess

import pytest

from oracle import oracle
from tests import (test_oracle_attention, test_oracle_fp8, test_oracle_fullc, test_oracle_linear,
                   test_oracle_modulate, test_oracle_norm_rope, test_oracle_rope3, test_oracle_skip)

MUTANTS = {
    "attn_drop_scale": ("s[j] = scale * acc;", "s[j] = acc;"),
    "attn_value_row_of_query": ("const int64_t vb = (lo + j) * stride_t", "const int64_t vb = t * stride_t"),
    "attn_lse_log2": ("lse[r * H + h] = m + log(l);", "lse[r * H + h] = m + log2(l);"),
    "attn_drop_last_key": ("L = (int64_t)cu[seg + 1] - cu[seg];", "L = (int64_t)cu[seg + 1] - cu[seg] - 1;"),
    "attn_no_normalise": ("ot[d] /= l;", "ot[d] /= 1.0;"),
    "attn_key_from_other_head": ("const int64_t kb = (lo + j) * stride_t + (int64_t)h * D;",
                                 "const int64_t kb = (lo + j) * stride_t;"),
    "rope_sign": ("out[ia] = a * cos(phi) - b * sin(phi);", "out[ia] = a * cos(phi) + b * sin(phi);"),
    "rope_exponent": ("pow(base, -2.0 * (double)j / (double)D)", "pow(base, -1.0 * (double)j / (double)D)"),
    "rope_pairing_swapped": ("if (style == ORACLE_ROPE_INTERLEAVED) { *ia = 2 * j;",
                             "if (style != ORACLE_ROPE_INTERLEAVED) { *ia = 2 * j;"),
    "norm_eps_outside_sqrt": ("ms /= (double)D;\n  const double inv = 1.0 / sqrt(ms + eps);",
                              "ms /= (double)D;\n  const double inv = 1.0 / (sqrt(ms) + eps);"),
    "fullc_eps_outside_sqrt": ("ms /= (double)width;\n    const double inv = 1.0 / sqrt(ms + eps);",
                               "ms /= (double)width;\n    const double inv = 1.0 / (sqrt(ms) + eps);"),
    "norm_sum_not_mean": ("ms /= (double)D;", "ms /= 1.0;"),
    "norm_drop_weight": ("n[d] = load(x, x_kind, row + d) * inv * load(w, w_kind, d);",
                         "n[d] = load(x, x_kind, row + d) * inv;"),
    "mod_scale_not_offset": ("n * (1.0 + (double)scale[", "n * (0.0 + (double)scale["),
    "mod_shift_of_first_request": ("+ (double)shift[(int64_t)seg * C + c];", "+ (double)shift[c];"),
    "mod_residual_sign": ("if (branch) xv += ", "if (branch) xv -= "),
    "mod_layer_unbiased": ("var /= (double)C;", "var /= (double)(C - 1);"),
    "mod_rms_mean_subtracted": ("n = xp[c] / sqrt(ms + eps);", "n = (xp[c] - mu) / sqrt(ms + eps);"),
    "silu_operands_swapped": ("act_out[r * (int64_t)F + f] = g / (1.0 + exp(-g)) * u;",
                              "act_out[r * (int64_t)F + f] = u / (1.0 + exp(-u)) * g;"),
    "silu_sign": ("g / (1.0 + exp(-g)) * u", "g / (1.0 + exp(g)) * u"),
    "rope3_axis_boundary": ("const int axis = j < sec[0] ? 0 :", "const int axis = j <= sec[0] ? 0 :"),
    "rope3_axes_swapped": ("(j < sec[0] + sec[1] ? 1 : 2)", "(j < sec[0] + sec[1] ? 2 : 1)"),
    "rope3_ids_of_first_token": ("(double)pos3[t * 3 + axis]", "(double)pos3[axis]"),
    "fullc_mean_over_one_head": ("ms /= (double)width;", "ms /= (double)D;"),
    "fullc_weight_of_first_head": ("* inv * load(w, w_kind, (int64_t)h * D + d);", "* inv * load(w, w_kind, d);"),
    "skip_first_row_decides": ("for (int64_t i = 0; i < nr && skip; ++i) {", "for (int64_t i = 0; i < 1 && skip; ++i) {"),
    "skip_key_block_doubled": ("double* tm = &tmax[i * nkb + j / kblock];", "double* tm = &tmax[i * nkb + j / (2 * kblock)];"),
    "skip_sampled_row_block_doubled": ("const int64_t r0 = lo + ((t - lo) / qrows) * qrows;",
                                       "const int64_t r0 = lo + ((t - lo) / (2 * qrows)) * (2 * qrows);"),
    "skip_threshold_sign": ("if (!(tmax[i * nkb + jb] < M - tau)) skip = 0;", "if (!(tmax[i * nkb + jb] < M + tau)) skip = 0;"),
    "skip_natural_log_units": ("const double u = scale * dot / log(2.0);", "const double u = scale * dot;"),
    "e4m3_ties_away_from_zero": ("const double r = rint(a / quantum) * quantum;",
                                 "const double r = round(a / quantum) * quantum;"),
    "e4m3_two_mantissa_bits": ("const double quantum = ldexp(1.0, e - 3);", "const double quantum = ldexp(1.0, e - 2);"),
    "fp8_k_dequantised_with_q_scale": ("kd[i] = e4m3_value(kc[i]) * (double)dq[H + h];",
                                       "kd[i] = e4m3_value(kc[i]) * (double)dq[h];"),
    "fp8_amax_of_first_token": ("    for (int64_t t = 0; t < T; ++t)\n      for (int d = 0; d < D; ++d) {\n        const float v = (float)fabs(",
                                "    for (int64_t t = 0; t < 1; ++t)\n      for (int d = 0; d < D; ++d) {\n        const float v = (float)fabs("),
    "fp8_range_240": ("const float inv = amax > 0.0f ? 448.0f / amax : 1.0f;\n    deq[h]",
                      "const float inv = amax > 0.0f ? 240.0f / amax : 1.0f;\n    deq[h]"),
    "fp8_prologue_range_240": ("const float inv = amax > 0.0f ? 448.0f / amax : 1.0f;\n    *deq_out",
                               "const float inv = amax > 0.0f ? 240.0f / amax : 1.0f;\n    *deq_out"),
    "fp8_p_not_quantised": ("\n    const double pq = e4m3_value(e4m3_code((float)pj));", "\n    const double pq = pj;"),
    "fp8_denominator_quantised": ("\n    den += pj;\n", "\n    den += pq;\n"),
    "fp8_reference_first_key": ("    s[j] = scale * dot;\n    if (s[j] > m) m = s[j];",
                                "    s[j] = scale * dot;\n    if (j == 0) m = s[j];"),
    "fp8_v_with_q_scale": ("xd[i][e] = e4m3_value(c8[e]) * (double)dq[(int64_t)i * H + (e / D) % H];",
                           "xd[i][e] = e4m3_value(c8[e]) * (double)dq[(e / D) % H];"),
    "fp8_online_threshold_zero": ("} else if (bmax > mrun + threshold) {", "} else if (bmax > mrun) {"),
    "fp8_online_p_not_quantised": ("\n      const double pq = e4m3_value(e4m3_code((float)pj));",
                                   "\n      const double pq = pj;"),
    "fp8_online_denominator_quantised": ("\n      den += pj;\n", "\n      den += pq;\n"),
    "fp8_online_numerator_not_rescaled": ("      for (int d = 0; d < D; ++d) num[d] *= alpha;\n", ""),
    "fp8_prologue_scale_without_sqrt_d": ("const float amax = sqrtf((float)D) * maxw;", "const float amax = maxw;"),
    "fp8_prologue_signed_weight_max": ("const float a = (float)fabs(load(w, w_kind, d));",
                                       "const float a = (float)load(w, w_kind, d);"),
    "fp8_skip_dropped_keys_summed": ("    if (keep && !keep[j / kblock]) continue;\n    const double pj", "    const double pj"),
    "fp8_online_dropped_keys_summed": ("      if (keep && !keep[j / skip_kblock]) continue;\n", ""),
    "linear_w_transposed": ("load(w, in_kind, (int64_t)n * K + k)", "load(w, in_kind, (int64_t)k * N + n)"),
    "linear_gate_of_first_request": ("(double)gate_res[(int64_t)seg * N + n] * y", "(double)gate_res[n] * y"),
    "linear_residual_sign": ("load(x, in_kind, t * N + n) + (double)gate_res", "load(x, in_kind, t * N + n) - (double)gate_res"),
    "linear_a_stride_ignored": ("y += load(a, in_kind, t * a_stride + k)", "y += load(a, in_kind, t * K + k)"),
    "linear_drop_last_k": ("for (int k = 0; k < K; ++k) y += ", "for (int k = 0; k < K - 1; ++k) y += "),
    "linear_swiglu_halves_swapped": ("act[r * (int64_t)F + f] = gv / (1.0 + exp(-gv)) * uv;",
                                     "act[r * (int64_t)F + f] = uv / (1.0 + exp(-uv)) * gv;"),
    "linear_swiglu_up_from_gate_rows": ("uv += av * load(w1, in_kind, ((int64_t)F + f) * K + k);",
                                        "uv += av * load(w1, in_kind, (int64_t)f * K + k);"),
    "skip_tile_counts_any_block": ("if (keep[((int64_t)h * nqb + b) * nkb + jb]) all = 0;",
                                   "if (!keep[((int64_t)h * nqb + b) * nkb + jb]) all = 0;"),
}


def _pin_calls():
    for mod in (test_oracle_attention, test_oracle_norm_rope, test_oracle_modulate, test_oracle_rope3,
                test_oracle_fullc, test_oracle_skip, test_oracle_fp8, test_oracle_linear):
        for name, fn in inspect.getmembers(mod, inspect.isfunction):
            if not name.startswith("test_") or fn.__module__ != mod.__name__:
                continue
            marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
            if not marks:
                yield f"{mod.__name__}.{name}", fn, {}
                continue
            names = [[n.strip() for n in m.args[0].split(",")] for m in marks]
            for combo in itertools.product(*[m.args[1] for m in marks]):
                kw = {}
                for ns, vals in zip(names, combo):
                    vals = vals if len(ns) > 1 else (vals,)
                    kw.update(dict(zip(ns, vals)))
                yield f"{mod.__name__}.{name}{kw}", fn, kw


def _killed(lib_path):
    saved = oracle._lib
    oracle._lib = oracle.load(lib_path)
    failures = []
    try:
        for label, fn, kw in _pin_calls():
            try:
                fn(**kw)
            except (AssertionError, ValueError):
                failures.append(label)
    finally:
        oracle._lib = saved
    return failures


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_mutant(mutant, tmp_path):
    old, new = MUTANTS[mutant]
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"mutation site for {mutant} not found exactly once"
    path = tmp_path / "m.c"
    path.write_text(src.replace(old, new))
    so = str(tmp_path / "libm.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", so, str(path), "-lm"])
    failures = _killed(so)
    assert failures, f"no pin rejects mutant {mutant}"


def test_unmutated_build_passes_every_pin(tmp_path):
    so = str(tmp_path / "lib0.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", so, oracle.SRC, "-lm"])
    assert _killed(so) == []
