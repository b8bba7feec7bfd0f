"""The seeded input generator (block_sparse_attention_41_b200/workloads.py) against its stated recipe.

The generator feeds both the oracle and the CUDA path, so a silent change in it would move every
stored threshold and parity case. These checks pin the recipe: determinism, exact bf16 values,
the positional feature worked out by hand at one grid point, the sink keys, the text + video
layout of the guidance pair, the rounding rule and the unit sampler.
"""
import math

import numpy as np
import pytest

from block_sparse_attention_41_b200 import workloads as wl


def test_round_to_bf16_is_nearest_even():
    one = 1.0
    ulp = 2.0 ** -7  # bf16 spacing in [1, 2)
    vals = np.array([one, one + ulp / 2, one + 3 * ulp / 2, one + 0.75 * ulp, -(one + ulp / 2), 3.0e38])
    got = wl.round_to_bf16(vals).astype(np.float64)
    assert got[0] == 1.0
    assert got[1] == 1.0                # tie: stays on the even mantissa
    assert got[2] == one + 2 * ulp      # tie: goes up to the even mantissa
    assert got[3] == one + ulp          # nearest
    assert got[4] == -1.0
    assert np.isfinite(got[5]) and abs(got[5] - 3.0e38) <= 2.0 ** -8 * 3.0e38  # large values stay finite


def test_positional_feature_recipe_at_one_grid_point():
    grid, d = (4, 5, 6), 18
    feat = wl.positional_feature(grid, d)
    assert feat.shape == (4 * 5 * 6, d)
    t, y, x = 1, 2, 3
    row = feat[t * 30 + y * 6 + x]  # x fastest
    pos = (t, y, x)
    for c in range(d):
        f = (0.25, 0.125, 0.0625)[(c // 3) % 3]
        fn = math.sin if (c // 9) % 2 == 0 else math.cos
        assert row[c] == pytest.approx(fn(2 * math.pi * f * pos[c % 3]), abs=1e-12), c
    assert row[0] == pytest.approx(1.0)   # sin(2 pi / 4 * 1)
    assert row[9] == pytest.approx(0.0)   # cos(2 pi / 4 * 1)


@pytest.mark.parametrize("name", ["tiny_f32_L1024", "small_dit_L8192"])
def test_head_tensors_are_deterministic_exact_and_distinct(name):
    w = wl.WORKLOADS[name]
    q, k, v = wl.head_tensors(w, 0, 1)
    q2, k2, v2 = wl.head_tensors(w, 0, 1)
    assert all(np.array_equal(a, b) for a, b in ((q, q2), (k, k2), (v, v2)))
    assert q.shape == (w.L, w.d) and q.dtype == np.float32
    if w.dtype == "bf16":
        assert all(np.array_equal(wl.round_to_bf16(a), a) for a in (q, k, v))
    q0, _, _ = wl.head_tensors(w, 0, 0)
    assert not np.array_equal(q0, q)
    # Q and K share the positional feature, V does not
    feat = wl.positional_feature(w.grid, w.d)
    assert np.corrcoef((q - k).ravel(), feat.ravel())[0, 1] < 0.05
    assert np.corrcoef(q.ravel(), feat.ravel())[0, 1] > 0.5


def test_sink_keys_are_boosted_on_every_channel():
    w = wl.WORKLOADS["video720p_L75600"]
    _, k, _ = wl.head_tensors(w, 0, 3)
    row_mean = k.astype(np.float64).mean(axis=1)
    assert w.n_sinks == 8 and int((row_mean > 3.0).sum()) == w.n_sinks


def test_guidance_pair_shares_the_video_part_and_not_the_text():
    w = wl.WORKLOADS["text_video_cfg_L33272"]
    a = wl.head_tensors(w, 0, 2)
    b = wl.head_tensors(w, 1, 2)
    for x, y in zip(a, b):
        assert np.array_equal(x[w.n_text:], y[w.n_text:])
        assert not np.array_equal(x[: w.n_text], y[: w.n_text])
    dens = wl.target_densities(w)
    assert dens.shape == (w.H,) and np.all((dens >= 0.05) & (dens <= 0.5))


def test_sample_units_are_distinct_sorted_and_in_range():
    w = wl.WORKLOADS["video720p_L75600"]
    u = wl.sample_units(w, 200, seed_offset=3)
    assert u == sorted(u) and len(set(u)) == 200 and u == wl.sample_units(w, 200, seed_offset=3)
    assert all(0 <= b < w.B and 0 <= h < w.H and 0 <= i < w.n_blocks for b, h, i in u)
    assert wl.sample_units(w, 200, seed_offset=4) != u
