"""Pins for the Deep Forcing oracle (rCM guide, strategy 4; readings DF1-DF4).

- a hand-enumerated stream (tests/golden/deep_forcing_s1_w4_b2_f2_c4.txt)
- a budget that holds every dropped token: the cache is the whole history at
  natural time indices, so the attention equals the unbounded policy's (which
  is pinned to brute-force full causal attention)
- no budget: the kept frames are the sliding window's, with the sink moved to
  sit right before the tail
- no holes: sink, region, tail and chunk occupy one contiguous time range
- the selection is a brute-force stable sort by (-score, pool index)
"""
import itertools
import os

import numpy as np
import pytest

import rc_synth
from oracle import DeepForcingOracle, OracleStream, PolicyOracle, top_c

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _parse_golden():
    rows = []
    with open(os.path.join(GOLDEN, "deep_forcing_s1_w4_b2_f2_c4.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = [p.strip() for p in line.split("|")]
            c = int(parts[0].split()[1])
            sc = parts[1].split()[1:]
            scores = None if sc == ["-"] else [float(x) for x in sc]
            sect = {}
            for p in parts[2:]:
                name, *items = p.split()
                sect[name] = [] if items == ["-"] else items
            rows.append((c, scores, sect))
    return rows


def _as_entries(kept):
    sink = sorted({(k.content, k.tau) for k in kept if k.region == "sink"})
    hist = sorted({(k.content, k.tau) for k in kept if k.region == "hist"})
    cur = sorted({(k.content, k.tau) for k in kept if k.region == "cur"})
    comp = [(k.content, k.tok, k.tau) for k in kept if k.region == "comp"]
    return sink, comp, hist, cur


def test_hand_enumerated_stream():
    df = DeepForcingOracle(chunk_frames=2, sink_frames=1, window_frames=4, budget_tokens=4, frame_seqlen=2)
    for c, scores, sect in _parse_golden():
        kept = df.step(2 * c, 2, pool_scores=scores)
        sink, comp, hist, cur = _as_entries(kept)
        want_frames = lambda key: [tuple(int(v) for v in it.split(":")) for it in sect[key]]
        assert sink == want_frames("sink"), c
        assert hist == want_frames("hist"), c
        assert cur == want_frames("cur"), c
        want_comp = []
        for it in sect["comp"]:
            ft, tau = it.split(":")
            g, t = ft.split(".")
            want_comp.append((int(g), int(t), int(tau)))
        assert comp == want_comp, c
        # a selection was needed exactly where the file lists scores
        assert (df.last_selection is not None) == (scores is not None)


def _tiny(policy, **kw):
    return rc_synth.WORKLOADS["tiny"].replace(policy=policy, grid_h=2, grid_w=3, heads=2, **kw)


def test_large_budget_equals_unbounded_attention():
    """With room for every dropped token nothing is ever left out: sink,
    region and tail hold the whole history at its own time indices."""
    chunks = 7
    w_df = _tiny(rc_synth.POLICY_DEEP_FORCING, sink_frames=1, window_frames=6, chunks=chunks,
                 df_budget_tokens=6 * 40)
    w_none = w_df.replace(policy=rc_synth.POLICY_NONE, window_frames=chunks * 3, df_budget_tokens=0)
    a, b = OracleStream(w_df), OracleStream(w_none)
    for c in range(chunks):
        ka = a.step(c, 0)
        b.step(c, 0)
        taus = {(k.content, k.tok): k.tau for k in ka}
        assert all(taus[(k.content, k.tok)] == k.tau for k in b.kept_tokens)
        assert len(ka) == len(b.kept_tokens)
        oa, ob = a.outputs(), b.outputs()
        np.testing.assert_allclose(oa["o"], ob["o"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(oa["lse"], ob["lse"], rtol=0, atol=1e-12)


def test_zero_budget_is_sliding_with_sink_moved_to_the_tail():
    S_f, W_f, B = 2, 6, 3
    df = DeepForcingOracle(B, S_f, W_f, 0, frame_seqlen=4)
    sl = PolicyOracle(rc_synth.POLICY_SLIDING, B, S_f, W_f)
    for c in range(12):
        kt = df.step(B * c, B)
        kf = sl.step(B * c, B)
        frames = []
        for k in kt:
            e = (k.content, k.region)
            if not frames or frames[-1] != e:
                frames.append(e)
        assert frames == [(k.content, k.region) for k in kf]
        g_t = max(S_f, B * c + B - W_f)
        for k in kt:
            if k.region == "sink":
                assert k.tau == g_t - S_f + k.content
            else:
                assert k.tau == k.content


@pytest.mark.parametrize("S_f,W_f,B,F,C", [(1, 4, 2, 2, 4), (3, 6, 3, 5, 20), (0, 7, 3, 3, 9), (2, 8, 4, 1, 3)])
def test_no_holes_and_footprint(S_f, W_f, B, F, C):
    rng = np.random.default_rng(S_f * 100 + C)
    df = DeepForcingOracle(B, S_f, W_f, C, frame_seqlen=F)
    dropped = 0
    for c in range(25):
        pool = df.next_pool_size(B)
        before = df.tail_start(df.end)
        kt = df.step(B * c, B, pool_scores=rng.random(pool))
        dropped += (df.tail_start(df.end) - before) * F
        n_comp = sum(1 for k in kt if k.region == "comp")
        assert n_comp == min(C, dropped)
        g0, end = B * c, df.end
        frames = min(S_f, g0) + max(0, g0 - df.tail_start(end)) + (end - g0)
        assert len(kt) == frames * F + n_comp
        taus = sorted({k.tau for k in kt})
        assert taus == list(range(taus[0], taus[0] + len(taus)))   # contiguous: no holes
        assert taus[-1] == df.end - 1
        # region tokens stay in time order of their sources
        comp = [(k.content, k.tok) for k in kt if k.region == "comp"]
        assert comp == sorted(comp)


def test_selection_is_stable_sort_by_score_then_index():
    rng = np.random.default_rng(5)
    for n in range(1, 9):
        for _ in range(20):
            s = rng.integers(0, 3, n).astype(float)   # many ties
            for C in range(0, n + 1):
                order = sorted(range(n), key=lambda i: (-s[i], i))[:C]
                assert list(top_c(s, np.arange(n), C)) == sorted(order)


def test_selection_must_be_given_when_the_pool_overflows():
    df = DeepForcingOracle(1, 0, 2, 1, frame_seqlen=1)
    df.step(0, 1)
    df.step(1, 1)
    df.step(2, 1)                # frame 0 leaves the tail: a pool of 1 fits the budget
    assert df.comp == [(0, 0)] and df.last_selection is None
    with pytest.raises(ValueError):
        df.step(3, 1)            # frame 1 leaves too: 2 tokens for 1 place, no scores
    df.step(3, 1, pool_scores=[0.1, 0.2])
    assert df.comp == [(1, 0)] and list(df.last_selection) == [1]
