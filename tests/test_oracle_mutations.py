"""Each pin must reject a copy of the oracle with a plausible mistake planted.

The mistakes are planted in oracle code on the CPU (monkeypatched copies);
nothing here touches the library or a GPU.
"""
import numpy as np
import pytest

import rc_synth

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


# ---- the policy oracles of the next rows: each pinned test file must reject
# a copy of its oracle with a plausible mistake planted.

import oracle.deep_forcing as odf
import oracle.memrope as omr
import oracle.relax_forcing as orf

import test_oracle_deep_forcing as tdf
import test_oracle_memrope as tmr
import test_oracle_relax_forcing as trf


def _rejected(*checks):
    """True when at least one of the pinned checks fails."""
    for fn, args in checks:
        try:
            fn(*args)
        except AssertionError:
            return True
    return False


def test_deep_forcing_pins_reject_region_time_off_by_one(monkeypatch):
    orig = odf.DeepForcingOracle.kept

    def kept(self):
        return [odf.KeptToken(k.content, k.tok, k.tau - 1, k.region, k.rank) if k.region == "comp" else k
                for k in orig(self)]
    monkeypatch.setattr(odf.DeepForcingOracle, "kept", kept)
    assert _rejected((tdf.test_hand_enumerated_stream, ()))


def test_deep_forcing_pins_reject_pool_without_leaving_frames(monkeypatch):
    # the pool forgets the frames leaving the tail: only the old region is ever re-selected
    orig_step = odf.DeepForcingOracle.step

    def step(self, frame_start, n_frames, pool_scores=None, selection=None):
        if self.cur_start is not None and frame_start == self.cur_start:
            return orig_step(self, frame_start, n_frames, pool_scores, selection)
        self.end = frame_start + n_frames
        self.cur_start, self.cur_n = frame_start, n_frames
        self.last_selection = None
        return self.kept()
    monkeypatch.setattr(odf.DeepForcingOracle, "step", step)
    assert _rejected((tdf.test_hand_enumerated_stream, ()))


def test_deep_forcing_pins_reject_ties_to_the_newer_token(monkeypatch):
    def ties_high(scores, idx, C):
        order = np.lexsort((-np.asarray(idx), -np.asarray(scores)))
        return np.sort(np.asarray(idx)[order[:C]])
    monkeypatch.setattr(odf, "top_c", ties_high)
    assert _rejected((tdf.test_hand_enumerated_stream, ()))


def test_relax_forcing_pins_reject_complement_sign(monkeypatch):
    def scores(pool_desc, tail_desc, weight):
        n = len(pool_desc)
        align = np.array([orf.cosine(d, tail_desc) for d in pool_desc])
        comp = np.ones(n)
        if n > 1:
            for i in range(n):
                comp[i] = 1.0 + sum(orf.cosine(pool_desc[i], pool_desc[j]) for j in range(n) if j != i) / (n - 1)
        return weight * align + (1.0 - weight) * comp
    monkeypatch.setattr(orf, "relax_scores", scores)
    assert _rejected((trf.test_hand_computed_stream, (0.5,)), (trf.test_hand_computed_stream, (0.9,)))


def test_relax_forcing_pins_reject_swapped_weights(monkeypatch):
    orig = orf.relax_scores
    monkeypatch.setattr(orf, "relax_scores", lambda p, t, w: orig(p, t, 1.0 - w))
    assert _rejected((trf.test_hand_computed_stream, (0.9,)))


def test_relax_forcing_pins_reject_ties_to_the_newer_frame(monkeypatch):
    def select(scores, K):
        order = sorted(range(len(scores)), key=lambda i: (-scores[i], -i))
        return sorted(order[:K])
    monkeypatch.setattr(orf, "select_frames", select)
    assert _rejected((trf.test_hand_computed_stream, (0.5,)), (trf.test_hand_computed_stream, (0.9,)))


def test_memrope_pins_reject_swapped_ema_weights(monkeypatch):
    class Swapped(omr.MemRopeOracle):
        def __init__(self, *a, **kw):
            super().__init__(*a, **kw)
            self.alpha = {m: 1.0 - v for m, v in self.alpha.items()}
    monkeypatch.setattr(tmr, "MemRopeOracle", Swapped)
    assert _rejected((tmr.test_hand_computed_memories, ()))


def test_memrope_pins_reject_long_memory_inside_the_sink(monkeypatch):
    orig = omr.MemRopeOracle.kept

    def kept(self):
        return [odf.KeptToken(k.content, k.tok, k.tau - 1, k.region, k.rank) if k.content == omr.MEM_LONG else k
                for k in orig(self)]
    monkeypatch.setattr(omr.MemRopeOracle, "kept", kept)
    assert _rejected((tmr.test_hand_computed_memories, ()))


def test_memrope_pins_reject_zero_initialised_memories(monkeypatch):
    # the first evicted frame folded into zero memories instead of initialising them
    orig_step = omr.MemRopeOracle.step

    def step(self, frame_start, n_frames):
        for m in (omr.MEM_LONG, omr.MEM_SHORT):
            if self.mem_k[m] is None:
                xk = self.raw_frame(0, 1)
                self.mem_k[m] = np.zeros_like(xk)
                self.mem_v[m] = np.zeros_like(self.raw_frame(0, 2))
        return orig_step(self, frame_start, n_frames)
    monkeypatch.setattr(omr.MemRopeOracle, "step", step)
    assert _rejected((tmr.test_hand_computed_memories, ()), (tmr.test_ema_closed_form_and_extremes, (0.3,)))


# ---- token scores and the in-chunk mask

def _scores_per_query(p_per_head, cols):
    # the mass each query gives the candidates, not the mass each candidate gets
    return sum(p[:, cols].sum(axis=1) for p in p_per_head)


def _scores_mean_over_heads(p_per_head, cols):
    return oatt.column_scores(p_per_head, cols) / len(p_per_head)


def _scores_first_head_only(p_per_head, cols):
    return oatt.column_scores(p_per_head[:1], cols)


def _scores_shifted_column(p_per_head, cols):
    n = p_per_head[0].shape[1]
    return oatt.column_scores(p_per_head, (np.asarray(cols) + 1) % n)


@pytest.mark.parametrize("fn", [_scores_per_query, _scores_mean_over_heads, _scores_first_head_only,
                                _scores_shifted_column])
def test_column_scores_pin_rejects(fn):
    with pytest.raises(AssertionError):
        pins.check_column_scores_autograd(fn)


import oracle.stream as ostream
import test_oracle_attention as tatt


def _vis_strict(query_rank, key_rank, mask_block_frames=1):
    # a frame no longer sees its own keys
    qr = np.asarray(query_rank)[:, None] // mask_block_frames
    kr = np.asarray(key_rank)[None, :]
    return (kr < 0) | ((kr // mask_block_frames) < qr)


def _vis_unblocked_keys(query_rank, key_rank, mask_block_frames=1):
    # the block size applied to the query side only
    qr = np.asarray(query_rank)[:, None] // mask_block_frames
    kr = np.asarray(key_rank)[None, :]
    return (kr < 0) | (kr <= qr)


@pytest.mark.parametrize("fn,mask_block", [(_vis_strict, 1), (_vis_unblocked_keys, 2)])
def test_visibility_pins_reject(fn, mask_block, monkeypatch):
    monkeypatch.setattr(ostream, "visibility", fn)
    with np.errstate(invalid="ignore"):   # the strict mask leaves the first frame's rows empty
        assert _rejected((tatt.test_window_covering_history_is_full_causal_attention,
                          (rc_synth.POLICY_SLIDING, mask_block)))


import test_oracle_policy as tpol


@pytest.mark.parametrize("fn", [
    lambda prev, new: opol.evicted_contents(new, prev),              # what arrived, not what left
    lambda prev, new: sorted({k.content for k in prev} - {k.content for k in new})[1:],  # one lost
])
def test_eviction_pin_rejects(fn):
    with pytest.raises(AssertionError):
        tpol.check_eviction_is_the_oldest_window_frames(fn)


def _grid_column_major(frame_seqlen, grid_w):
    # tokens walked down columns instead of along rows
    grid_h = frame_seqlen // grid_w
    n = np.arange(frame_seqlen)
    return n % grid_h, n // grid_h


def test_grid_positions_pin_rejects_column_major(monkeypatch):
    monkeypatch.setattr(ostream, "token_grid_positions", _grid_column_major)
    assert _rejected((tatt.test_window_covering_history_is_full_causal_attention,
                      (rc_synth.POLICY_SLIDING, 1)))
