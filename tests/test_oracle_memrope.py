"""Pins for the MemRoPE oracle (rCM guide, MemRoPE tip; readings MR1-MR3).

- hand-computed memories and positions (tests/golden/memrope_scalar.txt)
- the iterated EMA equals its closed form a^(n-1) X_1 + sum (1-a) a^(n-i) X_i
- alpha 0 keeps the last evicted frame, alpha 1 the first
- a window holding the whole history folds nothing and equals the unbounded policy
"""
import os

import numpy as np
import pytest

import rc_synth
from oracle import PolicyOracle
from oracle.memrope import MEM_LONG, MEM_SHORT, MemRopeOracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _scalar_frames(g, tid):
    x = np.array([[g, 1.0]]) if tid == 1 else np.array([[2.0 * g, -1.0 * g]])
    return x.reshape(1, 1, 2)


def test_hand_computed_memories():
    mr = MemRopeOracle(1, 0, 2, 0.5, 0.25, 1, _scalar_frames)
    rows = {}
    with open(os.path.join(GOLDEN, "memrope_scalar.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            p = [x.strip() for x in line.split("|")]
            c = int(p[0].split()[1])
            vec = lambda s: [float(v) for v in s.split(",")]
            lk, lv = p[2].split()[1], p[2].split()[3]
            sk, sv = p[3].split()[1], p[3].split()[3]
            rows[c] = (int(p[1].split()[1]), vec(lk), vec(lv), vec(sk), vec(sv),
                       [int(v) for v in p[4].split()[1:]])
    for c in range(5):
        kept = mr.step(c, 1)
        if c not in rows:
            assert not mr.folded
            continue
        ev, lk, lv, sk, sv, taus = rows[c]
        assert mr.folded[-1] == ev
        np.testing.assert_allclose(mr.memory(MEM_LONG, 1).reshape(-1), lk, atol=1e-15)
        np.testing.assert_allclose(mr.memory(MEM_LONG, 2).reshape(-1), lv, atol=1e-15)
        np.testing.assert_allclose(mr.memory(MEM_SHORT, 1).reshape(-1), sk, atol=1e-15)
        np.testing.assert_allclose(mr.memory(MEM_SHORT, 2).reshape(-1), sv, atol=1e-15)
        got = [k.tau for k in kept if k.content in (MEM_LONG, MEM_SHORT)]
        assert got == taus


@pytest.mark.parametrize("alpha", [0.0, 0.3, 0.9, 1.0])
def test_ema_closed_form_and_extremes(alpha):
    rng = np.random.default_rng(int(alpha * 10))
    frames = {g: rng.standard_normal((3, 2, 4)) for g in range(40)}
    mr = MemRopeOracle(2, 1, 4, alpha, alpha, 3, lambda g, tid: frames[g] * (1 if tid == 1 else -2))
    for c in range(15):
        mr.step(2 * c, 2)
    xs = [frames[g] for g in mr.folded]
    n = len(xs)
    want = alpha ** (n - 1) * xs[0] + sum((1 - alpha) * alpha ** (n - 1 - i) * xs[i] for i in range(1, n))
    np.testing.assert_allclose(mr.memory(MEM_LONG, 1), want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(mr.memory(MEM_SHORT, 2), -2 * want, rtol=1e-12, atol=1e-12)
    if alpha == 0.0:
        np.testing.assert_array_equal(mr.memory(MEM_LONG, 1), xs[-1])
    if alpha == 1.0:
        np.testing.assert_array_equal(mr.memory(MEM_LONG, 1), xs[0])
    assert mr.folded == list(range(1, 1 + n))    # the sink frame is never folded


def test_window_holding_history_folds_nothing():
    mr = MemRopeOracle(3, 1, 30, 0.5, 0.5, 2, lambda g, tid: np.ones((2, 1, 2)))
    none = PolicyOracle(rc_synth.POLICY_NONE, 3, 1, 1000)
    for c in range(10):
        kt = mr.step(3 * c, 3)
        kf = none.step(3 * c, 3)
        assert not mr.folded
        frames = []
        for k in kt:
            if not frames or frames[-1] != (k.content, k.tau, k.region):
                frames.append((k.content, k.tau, k.region))
        assert frames == [(k.content, k.tau, k.region) for k in kf]


def test_memory_positions_nonnegative_and_layout():
    mr = MemRopeOracle(3, 0, 6, 0.5, 0.5, 2, lambda g, tid: np.ones((2, 1, 2)) * g)
    for c in range(12):
        kt = mr.step(3 * c, 3)
        assert all(k.tau >= 0 for k in kt)
        g_w = max(0, 3 * c + 3 - 6)
        mem = [k for k in kt if k.content < 0]
        assert len(mem) == (4 if mr.folded else 0)
        if mr.folded:
            assert {k.tau for k in mem if k.content == MEM_LONG} == {0}
            assert {k.tau for k in mem if k.content == MEM_SHORT} == {g_w - 1}
