"""The seeded input recipe (CPU only): the synthetic tensors that stand in
for the pages' activations have the shapes, distributions and structure the
design notes state, are reproducible, and do not depend on how many host
threads drew them.
"""

import numpy as np
import pytest

from packed_attention_qk_b200 import workloads as wl


def test_bf16_rounding_is_round_to_nearest_even():
    # 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7: ties go to
    # the even mantissa (1); 1 + 3 * 2^-8 goes up to 1 + 2^-6 (even)
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], np.float32)
    back = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(x))
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0]


def test_streams_are_reproducible_and_independent_of_thread_count():
    a = wl._draw(7, "q", 3 * wl.CHUNK + 123, "normal", threads=1)
    b = wl._draw(7, "q", 3 * wl.CHUNK + 123, "normal", threads=4)
    assert np.array_equal(a, b)
    # one tensor's stream does not depend on which other tensors were drawn
    k1 = wl.bf16_normal(7, "k", (1000, 4))
    wl.bf16_normal(7, "v", (1000, 4))
    assert np.array_equal(k1, wl.bf16_normal(7, "k", (1000, 4)))
    assert not np.array_equal(k1, wl.bf16_normal(7, "v", (1000, 4)))
    assert not np.array_equal(k1, wl.bf16_normal(8, "k", (1000, 4)))


def test_distributions_of_the_recipe():
    n = 1 << 20
    act = wl.bf16_bits_to_f64(wl.bf16_normal(3, "x", (n,)))
    assert abs(act.mean()) < 5e-3 and abs(act.std() - 1.0) < 5e-3
    w = wl.bf16_bits_to_f64(wl.bf16_weight(3, "w_q", n))
    assert w.min() >= 0.5 and w.max() <= 1.5 and abs(w.mean() - 1.0) < 2e-3
    mod = wl.f32_modulation(3, "shift", (n,))
    assert mod.dtype == np.float32 and abs(mod.std() - 0.1) < 1e-3
    lw = wl.bf16_bits_to_f64(wl.bf16_linear_weight(3, "w1", 512, 2048))
    assert lw.shape == (512, 2048) and abs(lw.std() * np.sqrt(2048) - 1.0) < 5e-3


def test_outlier_variant_scales_about_one_in_a_thousand_by_twenty():
    shp = (4096, 2, 128)
    plain = wl.bf16_bits_to_f64(wl.bf16_normal(3, "k", shp))
    out = wl.bf16_bits_to_f64(wl.bf16_k_with_outliers(3, shp))
    changed = plain != out
    share = changed.mean()
    assert 0.0008 < share < 0.0012
    ratio = out[changed] / plain[changed]
    assert np.all(np.abs(ratio - 20.0) < 20.0 * 2 ** -7)   # x20 before one bf16 rounding


def test_configurations_match_their_descriptions():
    c1, c2, c3, c4 = (wl.config(i) for i in (1, 2, 3, 4))
    assert (c1.seg_lens, c1.H, c1.D, c1.C, c1.F) == ([200, 312], 4, 64, 256, 512)
    assert (c2.T, c2.H, c2.D, c2.C, c2.F) == (4096, 16, 128, 2048, 5632)
    assert (c3.T, c3.H, c3.D, c3.C, c3.F) == (58048, 24, 128, 3072, 8192)
    assert c4.seg_lens == [12345, 29024, 58048, 87072] and c4.T == 186489
    for T in wl.C5_TOKENS:
        c5 = wl.config(5, T)
        assert (c5.T, c5.H, c5.D, c5.C, c5.F) == (T, 40, 128, 5120, 13824)
    assert c3.attn_flops() == 4.0 * 24 * 128 * 58048 ** 2


def test_positions_restart_per_modality_and_video_ids_are_flattened():
    c3 = wl.config(3)
    pos = c3.positions()
    assert pos.dtype == np.int32 and pos.shape == (58048,)
    assert pos[0] == 0 and pos[511] == 511 and pos[512] == 0            # text, then audio restarts
    assert pos[512 + 2239] == 2239 and pos[2752] == 0                   # video restarts
    assert pos[-1] == 12 * 48 * 96 - 1
    p3 = c3.positions3()
    assert p3.shape == (58048, 3)
    t, h, w = 5, 17, 40
    row = 2752 + t * 48 * 96 + h * 96 + w
    assert p3[row].tolist() == [t, h, w] and pos[row] == t * 48 * 96 + h * 96 + w
    assert p3[100].tolist() == [100, 100, 100]                          # text ids repeated on the axes


def test_sampled_rows_include_each_requests_first_and_last_row():
    w = wl.custom([5, 0, 300, 1], 2, 64)
    rows = wl.sample_rows(w, per_segment=16)
    cu = w.cu_seqlens()
    for i in range(w.B):
        lo, hi = int(cu[i]), int(cu[i + 1])
        if hi > lo:
            assert lo in rows and hi - 1 in rows
            assert len([r for r in rows if lo <= r < hi]) == min(16, hi - lo)
    assert len(set(rows.tolist())) == len(rows)
    assert np.array_equal(rows, wl.sample_rows(w, per_segment=16))


def test_linear_inputs_shapes_and_gate_rows_first():
    w = wl.custom([100, 28], 2, 64, C=128, F=192, seed=3)
    o, w1, w2 = (wl.linear_inputs(w, n) for n in ("o_proj", "w1", "w2"))
    assert o["a"].shape == (128, 128) and o["w"].shape == (128, 128) and o["gate_res"].shape == (2, 128)
    assert w1["a"].shape == (128, 128) and w1["w"].shape == (384, 128) and set(w1) == {"a", "w"}
    assert w2["a"].shape == (128, 192) and w2["w"].shape == (128, 192) and np.array_equal(w2["x"], o["x"])
    with pytest.raises(ValueError):
        wl.linear_inputs(w, "qkv")


def test_batch_positions_reuse_the_joint_layout_for_its_58k_request():
    c4 = wl.config(4)
    pos = c4.positions()
    cu = c4.cu_seqlens()
    assert pos[cu[1] - 1] == 12344 and pos[cu[1]] == 0                 # 0..L-1 for plain requests
    third = pos[cu[2]:cu[3]]
    assert np.array_equal(third, wl.config(3).positions())              # text / audio / video runs of the 58k one
    assert pos[-1] == 87071
