"""The C++ policy engine (host-only handles) against the fp64 oracle's integer state.

Every step of every workload: kept (content, tau, region, rank) in logical
order must equal the oracle's bit for bit; the slot table must be a valid
ring mapping; eviction moves no bytes (slots of persisting frames stay put).
"""
import random

import pytest

import rc_synth
from oracle import PolicyOracle
from oracle.policy import evicted_contents
from rolling_kv_cache_b200 import binding as B

from rcutil import config_for, lib_kept, oracle_df_frames, oracle_kept


def run_df_stream(w, seed=0):
    """Deep Forcing: the engine plans the region by counts and times only
    (which tokens it holds is decided on the device), so the oracle gets
    arbitrary pool scores here and the frame list, region size and region
    time must match."""
    import numpy as np
    from oracle import DeepForcingOracle
    rng = np.random.default_rng(seed)
    cfg = config_for(w, layers=1)
    h = B.rc_cache_create(cfg, 0, 0)
    df = DeepForcingOracle(w.chunk_frames, w.sink_frames, w.window_frames, w.df_budget_tokens,
                           w.frame_seqlen)
    F = w.frame_seqlen
    n = 0
    prev_sink_tau = None
    try:
        for c, p, g0, cut in rc_synth.stream_schedule(w):
            B.rc_step(h, 0, 0, 0, 0, g0, w.chunk_frames, w.policy, 0)
            pool = rng.random(df.next_pool_size(w.chunk_frames)) if p == 0 else None
            kt = df.step(g0, w.chunk_frames, pool_scores=pool)
            st = B.rc_get_state(h, 0)
            frames = oracle_df_frames(kt)
            assert lib_kept(st) == frames, (c, p)
            sink_tau, tau0, V = df.frame_taus()
            assert st.comp_tokens == len(df.comp) == V * F
            if V:
                assert st.comp_tau0 == tau0
            assert st.valid_tokens == len(kt)
            assert st.n_candidates == sum(1 for k in kt if k.region in ("comp", "hist"))
            # keys carry their own time (no uniform shift); the sink moves only at new chunks
            assert all(e.stored_time == e.tau for e in st.kept[:st.n_kept])
            moved = (prev_sink_tau is not None and len(prev_sink_tau) == len(sink_tau)
                     and sink_tau != prev_sink_tau)
            if p > 0:
                assert st.n_jobs == 0
            elif moved:
                assert st.n_jobs >= 1
            prev_sink_tau = sink_tau
            n += 1
    finally:
        B.rc_cache_destroy(h)
    return n


def run_rf_stream(w, seed=0):
    """Relax Forcing: the engine plans the history region by counts only
    (which frames it holds is decided on the device from the descriptors), so
    the oracle gets arbitrary descriptors here; the sink / tail / chunk frames
    and the history size must match."""
    import numpy as np
    from oracle.relax_forcing import RelaxForcingOracle
    rng = np.random.default_rng(seed)
    desc = {}
    rf = RelaxForcingOracle(w.chunk_frames, w.sink_frames, w.window_frames, w.rf_history_frames,
                            w.rf_weight, lambda g: desc.setdefault(g, rng.standard_normal(4)))
    h = B.rc_cache_create(config_for(w, layers=1), 0, 0)
    F = w.frame_seqlen
    n = 0
    try:
        for c, p, g0, cut in rc_synth.stream_schedule(w):
            B.rc_step(h, 0, 0, 0, 0, g0, w.chunk_frames, w.policy, 0)
            kept = rf.step(g0, w.chunk_frames)
            st = B.rc_get_state(h, 0)
            hist = set(rf.hist)
            frames = [(k.content, k.tau, k.region, k.rank) for k in kept
                      if not (k.region == "hist" and k.content in hist)]
            assert lib_kept(st) == frames, (c, p)
            assert st.comp_tokens == len(rf.hist) * F
            assert st.valid_tokens == len(kept) * F
            assert st.n_jobs == 0      # nothing is re-rotated
            n += 1
    finally:
        B.rc_cache_destroy(h)
    return n


def run_mr_stream(w):
    """MemRoPE: sliding window plus the two memory frames (content -1 long at
    time S_f, -2 short right before the window) once a frame has left."""
    import numpy as np
    from oracle.memrope import MemRopeOracle
    mr = MemRopeOracle(w.chunk_frames, w.sink_frames, w.window_frames, w.mr_alpha_long,
                       w.mr_alpha_short, w.frame_seqlen, lambda g, tid: np.zeros((1, 1, 1)))
    h = B.rc_cache_create(config_for(w, layers=1), 0, 0)
    n = 0
    try:
        for c, p, g0, cut in rc_synth.stream_schedule(w):
            B.rc_step(h, 0, 0, 0, 0, g0, w.chunk_frames, w.policy, 0)
            kt = mr.step(g0, w.chunk_frames)
            st = B.rc_get_state(h, 0)
            assert lib_kept(st) == oracle_df_frames(kt), (c, p)
            assert st.valid_tokens == len(kt)
            P = w.sink_frames + w.window_frames
            for e in st.kept[:st.n_kept]:
                if e.content < 0:
                    assert e.slot == P + (0 if e.content == -1 else 1)
            assert st.n_jobs == 0
            n += 1
    finally:
        B.rc_cache_destroy(h)
    return n


def run_stream(w, steps=None):
    if w.policy == rc_synth.POLICY_MEMROPE:
        return run_mr_stream(w)
    if w.policy == rc_synth.POLICY_DEEP_FORCING:
        return run_df_stream(w)
    if w.policy == rc_synth.POLICY_RELAX_FORCING:
        return run_rf_stream(w)
    cfg = config_for(w, layers=1)
    h = B.rc_cache_create(cfg, 0, 0)
    pol = PolicyOracle.from_workload(w)
    P = w.footprint_frames
    prev_slots = {}
    prev_kept = []
    n = 0
    try:
        for c, p, g0, cut in rc_synth.stream_schedule(w):
            if cut:
                B.rc_reindex(h, w.policy, w.cut_delta, B.RC_REINDEX_FLUSH | B.RC_REINDEX_CUT)
                pol.reindex(1 | 2, w.cut_delta)
            B.rc_step(h, 0, 0, 0, 0, g0, w.chunk_frames, w.policy, 0)
            kept = pol.step(g0, w.chunk_frames)
            st = B.rc_get_state(h, 0)
            assert lib_kept(st) == oracle_kept(kept), (c, p)
            assert st.valid_tokens == len(kept) * w.frame_seqlen
            slots = [e.slot for e in st.kept[:st.n_kept]]
            assert len(set(slots)) == len(slots) and all(0 <= s < P for s in slots)
            for e in st.kept[:st.n_kept]:
                if e.region == 0:
                    assert e.slot < w.sink_frames
                assert e.stored_time == e.tau + st.shift
            # a frame that stays resident with the same content keeps its slot
            cur = {(e.content, e.region != 2): e.slot for e in st.kept[:st.n_kept]}
            for key, s in cur.items():
                if key in prev_slots and key[1] and w.policy != rc_synth.POLICY_ROLLING_SINK:
                    assert prev_slots[key] == s
            if p == 0:
                assert sorted(st.evicted[:st.n_evicted]) == evicted_contents(prev_kept, kept)
            prev_slots = {(e.content, True): e.slot for e in st.kept[:st.n_kept]}
            prev_kept = kept
            n += 1
            if steps and n >= steps:
                break
    finally:
        B.rc_cache_destroy(h)
    return n


@pytest.mark.parametrize("name", list(rc_synth.WORKLOADS))
def test_engine_matches_oracle_every_step(name):
    w = rc_synth.WORKLOADS[name]
    assert run_stream(w) == w.chunks * w.passes


def test_engine_rolling_sink_static_semantics():
    w = rc_synth.WORKLOADS["rolling_sink"].replace(rs_static_semantics=1, chunks=40)
    run_stream(w)


def test_engine_block_causal_mask_variant():
    w = rc_synth.WORKLOADS["tiny"].replace(mask_block_frames=3)
    run_stream(w)


def test_engine_jobs_for_policies():
    # Infinity-RoPE: sink re-rotated every step once shifting (rotate-copy from
    # its pristine copy); after a cut the kept last block is re-rotated in place.
    w = rc_synth.WORKLOADS["infinity_rope"]
    cfg = config_for(w, layers=1)
    h = B.rc_cache_create(cfg, 0, 0)
    jobs = []
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        if cut:
            B.rc_reindex(h, w.policy, 21, 3)
        B.rc_step(h, 0, 0, 0, 0, g0, 3, w.policy, 0)
        jobs.append(B.rc_get_state(h, 0).n_jobs)
    B.rc_cache_destroy(h)
    assert jobs[:7] == [0] * 7          # no shift before G'_end > f_limit
    assert jobs[7] == 3 and jobs[8] == 3 and jobs[26] == 3
    assert jobs[27] == 6 and jobs[28] == 6 and jobs[32] == 3
    # Rolling Sink: one bank block copied per step after K
    w = rc_synth.WORKLOADS["rolling_sink"]
    h = B.rc_cache_create(config_for(w, layers=1), 0, 0)
    jobs = []
    for c in range(30):
        B.rc_step(h, 0, 0, 0, 0, 3 * c, 3, w.policy, 0)
        jobs.append(B.rc_get_state(h, 0).n_jobs)
    B.rc_cache_destroy(h)
    assert jobs[:7] == [0] * 7 and all(j == 3 for j in jobs[7:])


def test_engine_repeat_passes_and_layers_independent():
    w = rc_synth.WORKLOADS["wan13b"]
    cfg = config_for(w, layers=3)
    h = B.rc_cache_create(cfg, 0, 0)
    try:
        for c in range(8):
            for p in range(5):
                for l in range(3):
                    B.rc_step(h, l, 0, 0, 0, 3 * c, 3, w.policy, 0)
                    st = B.rc_get_state(h, l)
                    if p > 0:
                        assert st.n_evicted == 0 and st.n_jobs == 0
        with pytest.raises(B.RcError) as e:
            B.rc_step(h, 0, 0, 0, 0, 3 * 6, 3, w.policy, 0)   # backwards
        assert e.value.status == B.RC_ESTATE
        assert B.rc_get_state(h, 0).chunk_start == 21         # unchanged by the failed call
    finally:
        B.rc_cache_destroy(h)


def test_engine_sink_reindex_sliding():
    w = rc_synth.WORKLOADS["tiny"].replace(sink_frames=2)
    cfg = config_for(w, layers=1)
    h = B.rc_cache_create(cfg, 0, 0)
    pol = PolicyOracle.from_workload(w)
    for c in range(12):
        if c in (4, 9):
            B.rc_reindex(h, w.policy, 5 if c == 4 else -2, B.RC_REINDEX_SINK)
            pol.reindex(4, 5 if c == 4 else -2)
        B.rc_step(h, 0, 0, 0, 0, 3 * c, 3, w.policy, 0)
        assert lib_kept(B.rc_get_state(h, 0)) == oracle_kept(pol.step(3 * c, 3))
    B.rc_cache_destroy(h)


def test_engine_fuzz_against_oracle():
    rng = random.Random(1234)
    for trial in range(60):
        B_ = rng.randint(1, 4)
        pol_kind = rng.choice([0, 1, 2, 3, 4, 5, 6])
        if pol_kind == 2:
            K = rng.randint(2, 7)
            S = rng.randint(1, K - 1)
            w = rc_synth.WORKLOADS["rolling_sink"].replace(
                chunk_frames=B_, rs_bank_blocks=K, rs_sink_blocks=S, sink_frames=S * B_,
                window_frames=(K - S + 1) * B_, chunks=rng.randint(1, 40),
                rs_static_semantics=rng.randint(0, 1))
        elif pol_kind == 3:
            Sb = rng.randint(0, 2)
            Cb = rng.randint(Sb + 1, Sb + 6)
            cuts = tuple(sorted(rng.sample(range(1, 40), rng.randint(0, 3))))
            w = rc_synth.WORKLOADS["infinity_rope"].replace(
                chunk_frames=B_, ir_sink_blocks=Sb, ir_cache_blocks=Cb, sink_frames=Sb * B_,
                window_frames=(Cb - Sb + 1) * B_, ir_f_limit=rng.randint(B_, 30),
                chunks=rng.randint(1, 40), cut_chunks=cuts, cut_delta=rng.randint(0, 25))
        elif pol_kind == 6:
            w = rc_synth.WORKLOADS["tiny"].replace(
                policy=rc_synth.POLICY_MEMROPE, grid_h=2, grid_w=2, chunk_frames=B_,
                sink_frames=rng.randint(0, 4), window_frames=rng.randint(B_, B_ + 6),
                mr_alpha_long=0.9, mr_alpha_short=0.5, chunks=rng.randint(1, 30), passes=rng.randint(1, 2))
        elif pol_kind == 5:
            w = rc_synth.WORKLOADS["tiny"].replace(
                policy=rc_synth.POLICY_RELAX_FORCING, grid_h=2, grid_w=2, chunk_frames=B_,
                sink_frames=rng.randint(0, 4), window_frames=rng.randint(B_, B_ + 6),
                rf_history_frames=rng.randint(0, 8), chunks=rng.randint(1, 30), passes=rng.randint(1, 2))
        elif pol_kind == 4:
            F = 4
            w = rc_synth.WORKLOADS["tiny"].replace(
                policy=rc_synth.POLICY_DEEP_FORCING, grid_h=2, grid_w=2, chunk_frames=B_,
                sink_frames=rng.randint(0, 4), window_frames=rng.randint(2 * B_, 2 * B_ + 6),
                df_budget_tokens=F * rng.randint(0, 8), chunks=rng.randint(1, 30),
                passes=rng.randint(1, 2))
        else:
            S_f = rng.randint(0, 5)
            W_f = rng.randint(B_, 20)
            chunks = rng.randint(1, 30)
            if pol_kind == 0:
                W_f = max(W_f, chunks * B_ - S_f + 1)
            w = rc_synth.WORKLOADS["tiny"].replace(
                policy=pol_kind, chunk_frames=B_, sink_frames=S_f, window_frames=W_f,
                chunks=chunks, passes=rng.randint(1, 3), mask_block_frames=rng.randint(1, 3))
        run_stream(w)


def test_engine_partial_chunks_sliding_against_oracle():
    """Sliding / unbounded chunks of 1..chunk_frames frames (the last block of a
    video, or a caller stepping single frames): state equals the oracle's."""
    rng = random.Random(77)
    for trial in range(40):
        B_ = rng.randint(1, 4)
        S_f = rng.randint(0, 3)
        W_f = rng.randint(B_, 10)
        w = rc_synth.WORKLOADS["tiny"].replace(chunk_frames=B_, sink_frames=S_f, window_frames=W_f)
        h = B.rc_cache_create(config_for(w, layers=1), 0, 0)
        pol = PolicyOracle.from_workload(w)
        g = 0
        try:
            for _ in range(rng.randint(1, 20)):
                n = rng.randint(1, B_)
                for _pass in range(rng.randint(1, 2)):
                    B.rc_step(h, 0, 0, 0, 0, g, n, w.policy, 0)
                    kept = pol.step(g, n)
                    st = B.rc_get_state(h, 0)
                    assert lib_kept(st) == oracle_kept(kept)
                    assert st.chunk_frames == n
                g += n
        finally:
            B.rc_cache_destroy(h)
