"""Each pin must reject a copy of the oracle with a plausible mistake planted.

The mistakes are planted in oracle code on the CPU (monkeypatched copies);
nothing here touches the library or a GPU.
"""
import numpy as np
import pytest

import oracle.attention as oatt
import oracle.policy as opol
import oracle.rope as orope

import pins


def _sin_sign_flipped(x, angles):
    return orope.rope_apply(x, -angles)


def _axes_swapped(t, h, w, d, theta):
    return orope.rope_angles(h, t, w, d, theta)


def _freq_off_by_one(t, h, w, d, theta):
    pt, ph, pw = orope.rope_pair_split(d)
    def f(n):
        j = np.arange(n, dtype=np.float64) + 1
        return theta ** (-2.0 * j / (2.0 * n))
    return np.concatenate([np.outer(t, f(pt)), np.outer(h, f(ph)), np.outer(w, f(pw))], axis=1)


@pytest.mark.parametrize("apply_fn,angles_fn", [
    (_sin_sign_flipped, orope.rope_angles),
    (orope.rope_apply, _axes_swapped),
    (orope.rope_apply, _freq_off_by_one),
])
def test_rope_pin_rejects(apply_fn, angles_fn):
    with pytest.raises(AssertionError):
        pins.check_rope_complex(angles_fn, apply_fn)


def _scale_by_d(q, k, v, vis):
    return oatt.masked_sdpa(q * np.sqrt(q.shape[1]) / q.shape[1], k, v, vis)


def _transposed_pv(q, k, v, vis):
    o, lse, p = oatt.masked_sdpa(q, k, v, vis)
    return (p @ v[::-1]), lse, p


def _mask_ignored(q, k, v, vis):
    return oatt.masked_sdpa(q, k, v, np.ones_like(vis))


@pytest.mark.parametrize("fn", [_scale_by_d, _transposed_pv, _mask_ignored])
def test_sdpa_pin_rejects(fn):
    with pytest.raises(AssertionError):
        pins.check_sdpa_vs_torch(fn)


def test_topc_pin_rejects_wrong_tie_break():
    def ties_high(scores, idx, C):
        order = np.lexsort((-np.asarray(idx), -np.asarray(scores)))
        return np.sort(np.asarray(idx)[order[:C]])
    with pytest.raises(AssertionError):
        pins.check_topc_bruteforce(ties_high)


def test_rolling_sink_pin_rejects(monkeypatch):
    # roll without repeating the end block (period 2K-1)
    def roll_no_repeat(p, K):
        q = p % (2 * K - 2)
        return q if q < K else 2 * K - 2 - q
    monkeypatch.setattr(opol, "roll_index", roll_no_repeat)
    with pytest.raises(AssertionError):
        pins.check_rolling_sink(opol.PolicyOracle)


def test_rolling_sink_pin_rejects_segment_offset(monkeypatch):
    orig = opol.roll_index
    monkeypatch.setattr(opol, "roll_index", lambda p, K: orig(p + 1, K))
    with pytest.raises(AssertionError):
        pins.check_rolling_sink(opol.PolicyOracle)


def test_infinity_rope_pin_rejects(monkeypatch):
    class NoClamp(opol.PolicyOracle):
        def _infinity_rope(self, g0, n):
            out = super()._infinity_rope(g0, n)
            g_end_v = self.vtime[g0 + n - 1] + 1
            shift = max(0, g_end_v - self.f_limit)
            return [opol.KeptFrame(k.content, self.vtime[k.content] - shift, k.region, k.rank)
                    for k in out]
    with pytest.raises(AssertionError):
        pins.check_infinity_rope(NoClamp)

    class FlushDropsLastBlock(opol.PolicyOracle):
        def reindex(self, flags, t_delta):
            super().reindex(flags, t_delta)
            if flags & 1:
                self.flush_points[-1] += self.B
    with pytest.raises(AssertionError):
        pins.check_infinity_rope(FlushDropsLastBlock)


def test_lingbot_pin_rejects_window_off_by_one():
    class Wider(opol.PolicyOracle):
        def _sliding(self, g0, n, window):
            return super()._sliding(g0, n, window + 1)
    with pytest.raises(AssertionError):
        pins.check_lingbot_numbers(Wider, 1560, 6, 12, 3, 30)
