"""Pins for the oracle's 3D RoPE."""
import numpy as np
import pytest

from oracle import rope_angles, rope_apply, rope_pair_split, token_grid_positions

import pins


def test_pair_split_matches_config_dims():
    # Wan-1.3B workload text: RoPE t:44/h:42/w:42 dims at head_dim 128.
    pt, ph, pw = rope_pair_split(128)
    assert (2 * pt, 2 * ph, 2 * pw) == (44, 42, 42)
    # tiny workload (head_dim 64): reading R1 gives 12/10/10 pairs.
    assert rope_pair_split(64) == (12, 10, 10)


@pytest.mark.parametrize("d", [64, 128])
def test_complex_formulation(d):
    pins.check_rope_complex(rope_angles, rope_apply, head_dim=d)


def _rand(n, d, seed=1):
    return np.random.default_rng(seed).standard_normal((n, 3, d))


def test_norm_preserved_and_identity():
    x = _rand(11, 128)
    t = np.arange(11) * 37
    a = rope_angles(t, t % 30, t % 52, 128, 1e4)
    y = rope_apply(x, a)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-12)
    z = rope_apply(x, rope_angles(0 * t, 0 * t, 0 * t, 128, 1e4))
    assert np.array_equal(z, x)


def test_composition_and_inverse():
    x = _rand(9, 128)
    rng = np.random.default_rng(3)
    t1, t2 = rng.integers(0, 500, 9), rng.integers(-200, 200, 9)
    h, w = rng.integers(0, 30, 9), rng.integers(0, 52, 9)
    a1 = rope_angles(t1, h, w, 128, 1e4)
    a2 = rope_angles(t2, 0 * h, 0 * w, 128, 1e4)
    both = rope_angles(t1 + t2, h, w, 128, 1e4)
    assert np.allclose(rope_apply(rope_apply(x, a1), a2), rope_apply(x, both), atol=1e-10)
    assert np.allclose(rope_apply(rope_apply(x, a2), -a2), x, atol=1e-12)


def test_axes_touch_only_their_pairs():
    pt, ph, pw = rope_pair_split(128)
    x = _rand(4, 128)
    base = rope_apply(x, rope_angles([5] * 4, [3] * 4, [7] * 4, 128, 1e4))
    for axis, (lo, hi) in enumerate(((0, pt), (pt, pt + ph), (pt + ph, pt + ph + pw))):
        pos = [[5] * 4, [3] * 4, [7] * 4]
        pos[axis] = [9] * 4
        y = rope_apply(x, rope_angles(*pos, 128, 1e4))
        diff = np.abs(y - base).reshape(4, 3, 64, 2).max(axis=(0, 1, 3))
        changed = np.nonzero(diff > 1e-12)[0]
        assert list(changed) == list(range(lo, hi))


def test_grid_positions_row_major():
    hh, ww = token_grid_positions(1560, 52)
    assert hh.max() == 29 and ww.max() == 51
    assert (hh[53], ww[53]) == (1, 1)
