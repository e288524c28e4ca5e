"""Pins for the oracle's cache policies (integer state)."""
import pytest

import rc_synth
from oracle import PolicyOracle, roll_index
from oracle.policy import evicted_contents

import pins


def test_rolling_sink_hand_enumeration():
    pins.check_rolling_sink(PolicyOracle)


def test_roll_sequence_forward_then_reverse():
    # Rolling Sink digest, method-step details: forward on even cycles, reversed on odd.
    assert [roll_index(p, 6) for p in range(24)] == \
        [0, 1, 2, 3, 4, 5, 5, 4, 3, 2, 1, 0] * 2


def test_rolling_sink_content_period():
    B, K, S = 3, 6, 5
    pol = PolicyOracle(2, B, S * B, (K - S + 1) * B, rs_bank_blocks=K, rs_sink_blocks=S)
    seq = [[k.content for k in pol.step(i * B, B) if k.region == "sink"] for i in range(60)]
    for i in range(K, 60 - 2 * K):
        assert seq[i] == seq[i + 2 * K]


def test_rolling_sink_static_semantics():
    # Stage 2 (sliding indices): sink shows blocks 0..S-1 at times [i-K, i-K+S).
    B, K, S = 3, 6, 5
    pol = PolicyOracle(2, B, S * B, (K - S + 1) * B, rs_bank_blocks=K, rs_sink_blocks=S,
                       rs_static_semantics=1)
    for i in range(30):
        kept = pol.step(i * B, B)
        sink = [k for k in kept if k.region == "sink"]
        if i >= K:
            assert [(k.content, k.tau) for k in sink] == \
                [(j * B + o, (i - K + j) * B + o) for j in range(S) for o in range(B)]


def test_infinity_rope_hand_table():
    pins.check_infinity_rope(PolicyOracle)


def test_lingbot_worked_numbers():
    w = rc_synth.WORKLOADS["large"]
    pins.check_lingbot_numbers(PolicyOracle, w.frame_seqlen, w.sink_frames,
                               w.window_frames, w.chunk_frames, w.chunks)



def check_eviction_is_the_oldest_window_frames(evicted_fn):
    """LingBot's cache (sink + window frames) at steady state drops, per
    chunk, the chunk's worth of oldest non-sink frames it held before: 3
    frames = 4680 tokens at 1560-token frames, as its worked numbers say."""
    w = rc_synth.WORKLOADS["large"]
    B, S, W, F = w.chunk_frames, w.sink_frames, w.window_frames, w.frame_seqlen
    pol = PolicyOracle(1, B, S, W)
    prev, steady = None, 0
    for c in range(w.chunks + 6):
        kept = pol.step(c * B, B)
        if prev is not None:
            ev = list(evicted_fn(prev, kept))
            older = sorted(k.content for k in prev if k.region != "sink")
            if len(prev) == S + W:
                assert ev == older[:B]
                assert len(ev) * F == 4680
                steady += 1
            else:
                assert ev == []
        prev = kept
    assert steady >= 1


def test_evicted_contents_are_the_oldest_window_frames():
    check_eviction_is_the_oldest_window_frames(evicted_contents)


FRAME_POLICIES = [n for n, w in rc_synth.WORKLOADS.items()
                  if w.policy not in (rc_synth.POLICY_DEEP_FORCING, rc_synth.POLICY_RELAX_FORCING,
                                      rc_synth.POLICY_MEMROPE)]


@pytest.mark.parametrize("name", FRAME_POLICIES)
def test_footprint_constant(name):
    """valid tokens = min(history, footprint) every step; never more.
    (Deep / Relax Forcing footprints are pinned in test_oracle_deep_forcing.py /
    test_oracle_relax_forcing.py.)"""
    w = rc_synth.WORKLOADS[name]
    pol = PolicyOracle.from_workload(w)
    P = w.footprint_frames
    last_flush = -10 ** 9
    steady = {"tiny": 112, "wan13b": 29640, "large": 28080,
              "rolling_sink": 32760, "infinity_rope": 32760}[name]
    assert w.footprint_tokens == steady
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        if cut:
            pol.reindex(1 | 2, w.cut_delta)
            last_flush = c
        kept = pol.step(g0, w.chunk_frames)
        assert len(kept) <= P
        assert len({(k.content, k.tau, k.region) for k in kept}) == len(kept)
        if c - last_flush >= w.ir_cache_blocks:
            assert len(kept) == min(g0 + w.chunk_frames, P)
    assert len(kept) * w.frame_seqlen == steady


def test_repeat_pass_overwrites_and_evicts_nothing():
    w = rc_synth.WORKLOADS["wan13b"]
    pol = PolicyOracle.from_workload(w)
    for c in range(10):
        first = pol.step(3 * c, 3)
        for _ in range(4):
            again = pol.step(3 * c, 3)
            assert again == first
            assert evicted_contents(first, again) == []


def test_sliding_window_covering_history_is_unbounded_policy():
    B, S_f = 3, 1
    big = PolicyOracle(1, B, S_f, 300)
    none = PolicyOracle(0, B, S_f, 300)
    for c in range(50):
        a = big.step(3 * c, 3)
        b = none.step(3 * c, 3)
        assert [(k.content, k.tau, k.rank) for k in a] == [(k.content, k.tau, k.rank) for k in b]
        assert [k.content for k in a] == list(range(3 * c + 3))
        assert all(k.tau == k.content for k in a)


def test_sliding_sink_shift():
    pol = PolicyOracle(1, 3, 2, 6)
    for c in range(5):
        pol.step(3 * c, 3)
    pol.reindex(4, 7)
    kept = pol.step(15, 3)
    assert [(k.content, k.tau) for k in kept if k.region == "sink"] == [(0, 7), (1, 8)]
    assert [(k.content, k.tau) for k in kept if k.region != "sink"] == [(g, g) for g in range(12, 18)]


def test_errors():
    pol = PolicyOracle(1, 3, 1, 6)
    pol.step(0, 3)
    with pytest.raises(ValueError):
        pol.step(6, 3)          # gap
    pol.step(3, 3)
    with pytest.raises(ValueError):
        pol.step(0, 3)          # backwards
    with pytest.raises(ValueError):
        pol.step(3, 2)          # repeat with a different size
    rs = PolicyOracle(2, 3, 15, 6, rs_bank_blocks=6, rs_sink_blocks=5)
    with pytest.raises(ValueError):
        rs.step(0, 2)           # not a whole block
    with pytest.raises(ValueError):
        PolicyOracle(0, 3, 1, 5).step(0, 9)   # unbounded cache too small
