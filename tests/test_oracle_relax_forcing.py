"""Pins for the Relax Forcing oracle (rCM guide, strategy 5; readings RF1-RF6).

- hand-computed scores and selections (tests/golden/relax_forcing_2d.txt),
  including exact ties resolved to the older frame
- w = 1 keeps the frames most aligned with the tail, w = 0 the least
  redundant ones (brute force over the pool)
- cosine scores are invariant to scaling a descriptor and permute with the pool
- a history budget holding every dropped frame reproduces the unbounded
  policy (same frames, same time indices)
"""
import os

import numpy as np
import pytest

import rc_synth
from oracle import PolicyOracle
from oracle.relax_forcing import RelaxForcingOracle, frame_descriptor, relax_scores, select_frames

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
D2 = {0: (1, 0), 1: (0, 1), 2: (1, 1), 3: (1, 0), 4: (0, 1), 5: (2, 0)}


def _golden():
    out = []
    with open(os.path.join(GOLDEN, "relax_forcing_2d.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            p = [x.split() for x in line.split("|")]
            out.append((float(p[0][1]), int(p[1][1]), [int(v) for v in p[2][1:]],
                        [float(v) for v in p[3][1:]], [int(v) for v in p[4][1:]]))
    return out


@pytest.mark.parametrize("weight", [0.5, 0.9])
def test_hand_computed_stream(weight):
    rf = RelaxForcingOracle(1, 0, 2, 2, weight, lambda g: np.array(D2[g], dtype=np.float64))
    rows = {c: (pool, sc, keep) for w, c, pool, sc, keep in _golden() if w == weight}
    for c in range(6):
        rf.step(c, 1)
        if c in rows:
            pool, sc, keep = rows[c]
            assert rf.last_pool == pool
            np.testing.assert_allclose(rf.last_scores, sc, atol=6e-5)
            assert rf.last_selection == keep
            assert rf.hist == [pool[i] for i in keep]
        else:
            assert rf.last_scores is None


def test_weight_extremes_brute_force():
    rng = np.random.default_rng(1)
    for _ in range(30):
        n, K = rng.integers(3, 9), None
        K = int(rng.integers(1, n))
        descs = [rng.standard_normal(6) for _ in range(n)]
        tail = rng.standard_normal(6)
        cos = lambda a, b: float(a @ b / np.linalg.norm(a) / np.linalg.norm(b))
        s1 = relax_scores(descs, tail, 1.0)
        np.testing.assert_allclose(s1, [cos(d, tail) for d in descs], rtol=0, atol=1e-12)
        s0 = relax_scores(descs, tail, 0.0)
        want = [1 - np.mean([cos(descs[i], descs[j]) for j in range(n) if j != i]) for i in range(n)]
        np.testing.assert_allclose(s0, want, rtol=0, atol=1e-12)
        for s in (s0, s1):
            sel = select_frames(s, K)
            best = sorted(range(n), key=lambda i: (-s[i], i))[:K]
            assert sel == sorted(best)


def test_scale_invariance_and_permutation():
    rng = np.random.default_rng(2)
    descs = [rng.standard_normal(8) for _ in range(6)]
    tail = rng.standard_normal(8)
    s = relax_scores(descs, tail, 0.3)
    scaled = [d * (i + 0.5) for i, d in enumerate(descs)]
    np.testing.assert_allclose(relax_scores(scaled, 7.0 * tail, 0.3), s, rtol=0, atol=1e-12)
    perm = rng.permutation(6)
    np.testing.assert_allclose(relax_scores([descs[i] for i in perm], tail, 0.3), s[perm], rtol=0, atol=1e-12)


def test_frame_descriptor_is_token_mean_per_head():
    x = np.arange(2 * 3 * 4, dtype=np.float64).reshape(2, 3, 4)   # [F=2, H=3, d=4]
    d = frame_descriptor(x)
    np.testing.assert_array_equal(d, ((x[0] + x[1]) / 2).reshape(-1))


def test_large_history_equals_unbounded():
    B, S_f, W_f = 3, 1, 6
    rf = RelaxForcingOracle(B, S_f, W_f, 100, 0.5, lambda g: np.ones(4))
    none = PolicyOracle(rc_synth.POLICY_NONE, B, S_f, 1000)
    for c in range(15):
        a = rf.step(B * c, B)
        b = none.step(B * c, B)
        assert [(k.content, k.tau, k.region) for k in a] == [(k.content, k.tau, k.region) for k in b]
        assert rf.last_scores is None


def test_history_bounded_and_time_ordered():
    rng = np.random.default_rng(3)
    desc = {}
    rf = RelaxForcingOracle(3, 2, 6, 4, 0.5, lambda g: desc.setdefault(g, rng.standard_normal(5)))
    for c in range(20):
        kept = rf.step(3 * c, 3)
        assert len(rf.hist) <= 4 and rf.hist == sorted(rf.hist)
        assert all(k.tau == k.content for k in kept)
        assert len(kept) <= 2 + 4 + 6
