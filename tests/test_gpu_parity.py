"""GPU parity: the library (through its C ABI) against the fp64 oracle.

Integer state is compared bit for bit on every step; K/V appends and
re-rotations bit for bit against a CPU fp32 restatement of the kernels'
arithmetic; O / LSE against fp64 within max-abs 2e-2, mean-abs 2e-3 (O) and
1e-2 (LSE); scores within SCORE_TOL (2^-9, the bf16 unit roundoff) of the
largest; top-C exactly on the kernel's own scores and up to near-ties against
fp64.
"""
import numpy as np
import pytest
import torch

import rc_synth
from oracle import top_c
from rolling_kv_cache_b200 import binding as B
from rolling_kv_cache_b200.cache import RollingKVCache

from gpu_util import Runner, bits_of, dev_bf16, rope_fp32, rope_fp32_delta
from rcutil import SCORE_TOL, config_for, near_tie_violations

pytestmark = pytest.mark.gpu

W = rc_synth.WORKLOADS


def test_watchdog_reports_timeout_and_context_survives():
    w = W["tiny"]
    cache = RollingKVCache(config_for(w))
    cache.watchdog_selftest(20000)
    with pytest.raises(B.RcError) as e:
        cache.device_status()
    assert e.value.status == B.RC_ETIMEOUT
    q, k, v = (dev_bf16(x) for x in rc_synth.chunk_qkv(w, 0, 0, 0))
    out = cache.step(0, q, k, v, 0)
    torch.cuda.synchronize()
    cache.device_status()           # cleared, and the context still works
    assert torch.isfinite(out.float()).all()
    cache.close()


@pytest.mark.parametrize("mask_block", [1, 3])
def test_tiny_every_step(mask_block):
    w = W["tiny"].replace(mask_block_frames=mask_block)
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p, cut)
        r.check_append_bitexact()
        r.check_float()
    r.close()


@pytest.mark.parametrize("sink,window,grid,heads,d", [
    (0, 3, (4, 4), 2, 64),      # no sink, window = one chunk: attention over the chunk only
    (2, 4, (10, 10), 1, 64),    # one history frame, 100-token frames (ragged tiles), one head
    (1, 6, (3, 50), 3, 128),    # 150-token frames: tiles straddle frame boundaries
])
def test_degenerate_and_ragged_configs(sink, window, grid, heads, d):
    w = W["tiny"].replace(sink_frames=sink, window_frames=window, grid_h=grid[0], grid_w=grid[1],
                          heads=heads, head_dim=d, chunks=7)
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p)
        r.check_append_bitexact()
        r.check_float()
    r.close()


def test_unbounded_policy_equals_full_history():
    w = W["tiny"].replace(policy=rc_synth.POLICY_NONE, window_frames=40, chunks=8)
    r = Runner(w)
    for c in range(w.chunks):
        r.step(c, 0)
        r.check_float()
    r.close()


@pytest.mark.parametrize("mask_block", [1, 3])
def test_multi_tile_ragged(mask_block):
    # F = 200 tokens: a frame is 1.56 tiles, Nq = 600 = 4 tiles + 88 rows,
    # cache runs end mid-tile; 3 heads of 128.
    w = rc_synth.Workload(name="ragged", workload_id=11, layers=1, heads=3, head_dim=128, grid_h=10,
                          grid_w=20, chunk_frames=3, sink_frames=1, window_frames=6,
                          policy=rc_synth.POLICY_SLIDING, chunks=6, dist="normal_frame_mean",
                          mask_block_frames=mask_block)
    r = Runner(w)
    for c in range(w.chunks):
        r.step(c, 0)
        r.check_append_bitexact()
        r.check_float()
    r.close()


@pytest.mark.parametrize("mask_block,d", [(1, 128), (3, 128), (1, 64)])
def test_stream_k_split_units(mask_block, d):
    # 64 heads x 3 query pairs = 192 (head, pair) units > 148 SMs: the
    # persistent schedule splits units between CTAs and the combine kernel
    # merges their partial rows (and drops their L2 lines, four threads to a
    # line at d = 64, two at d = 128). 240-token frames keep tiles ragged.
    w = rc_synth.Workload(name="streamk", workload_id=13, layers=1, heads=64, head_dim=d, grid_h=12,
                          grid_w=20, chunk_frames=3, sink_frames=1, window_frames=6,
                          policy=rc_synth.POLICY_SLIDING, chunks=4, mask_block_frames=mask_block)
    r = Runner(w)
    for c in range(w.chunks):
        r.step(c, 0)
        r.check_float()
    r.close()


def test_host_pipeline_matches_device_path():
    # pinned host buffers through the overlapped upload/compute/download
    # pipeline give the same bytes as device tensors through rc_step
    w = W["tiny"].replace(heads=4, head_dim=128, grid_h=8, grid_w=16, passes=2, chunks=5)
    a = RollingKVCache(config_for(w))
    b = RollingKVCache(config_for(w))
    pipe = b.host_pipeline(depth=2)
    outs_a, outs_b = [], []
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        q, k, v = rc_synth.chunk_qkv(w, 0, c, p)
        outs_a.append(bits_of(a.step(0, dev_bf16(q), dev_bf16(k), dev_bf16(v), g0)))
        hq, hk, hv = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (q, k, v))
        ob = torch.empty(hq.shape, dtype=torch.bfloat16, pin_memory=True)
        pipe.submit(0, hq, hk, hv, g0, ob)
        outs_b.append(ob)
    pipe.synchronize()
    for oa, ob in zip(outs_a, outs_b):
        assert np.array_equal(oa, ob.view(torch.int16).numpy().view(np.uint16))
    a.close()
    b.close()


def test_repeat_passes_overwrite():
    w = rc_synth.Workload(name="passes", workload_id=12, layers=2, heads=2, head_dim=128, grid_h=8,
                          grid_w=16, chunk_frames=3, sink_frames=1, window_frames=9,
                          policy=rc_synth.POLICY_SLIDING, chunks=6, passes=3, dist="normal_frame_mean")
    r = Runner(w, layer=1)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p)
        r.check_float()
    r.close()


def test_rolling_sink_small():
    w = W["rolling_sink"].replace(heads=2, grid_h=8, grid_w=8, chunks=16)
    r = Runner(w)
    for c in range(w.chunks):
        r.step(c, 0)
        r.check_append_bitexact()
        r.check_float()
        st = r.last["state"]
        if c >= 7:   # the entering sink block was rotate-copied from the bank
            kc, vc = r.cache.cache_views(0)
            rk, rv = r.cache.raw_views(0)
            F = w.frame_seqlen
            n = np.arange(F)
            for e in st.kept[:st.n_kept]:
                if e.region != 0:
                    continue
                got = bits_of(kc[:, e.slot * F:(e.slot + 1) * F]).transpose(1, 0, 2)
                raw = bits_of(rk[:, e.content * F:(e.content + 1) * F]).transpose(1, 0, 2)
                want = rope_fp32(raw, np.full(F, e.stored_time), n // w.grid_w, n % w.grid_w,
                                 r.tables, r.pairs)
                assert np.array_equal(got, want)
                gv = bits_of(vc[:, e.slot * F:(e.slot + 1) * F])
                assert np.array_equal(gv, bits_of(rv[:, e.content * F:(e.content + 1) * F]))
    r.close()


def _topc_checks(w, r, ref):
    sg = r.last["scores"]
    sr = ref["scores"]
    assert len(sg) == len(sr)
    if len(sr) == 0:   # no history yet: nothing to score, top-C all -1
        assert np.all(r.last["topc"] == -1)
        return
    rel = np.abs(sg - sr) / np.maximum(np.abs(sr), 1e-30)
    assert np.max(np.abs(sg - sr)) <= SCORE_TOL * max(1.0, np.max(np.abs(sr))), np.max(rel)
    cand = ref["cand_index"]
    # (i) selection on the kernel's own fp32 scores is exact
    want = top_c(sg.astype(np.float32), cand, w.topc)
    got = r.last["topc"]
    n = min(w.topc, len(cand))
    assert np.array_equal(got[:n], want)
    assert np.all(got[n:] == -1)
    # (ii) against the fp64 selection, swaps only among near-ties of the C-th score
    if n < len(cand):
        pos = {int(c): i for i, c in enumerate(cand)}
        bad = near_tie_violations(sr, [pos[int(c)] for c in got[:n]], n)
        assert not bad, bad[:8]
    else:
        assert np.array_equal(np.sort(ref["topc"]), got[:n])


@pytest.mark.parametrize("d", [128, 64])
def test_infinity_rope_small_with_scores(d):
    w = W["infinity_rope"].replace(heads=2, head_dim=d, grid_h=8, grid_w=8, chunks=18, cut_chunks=(9, 13),
                                   topc=100)
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p, cut, scores=True)
        r.check_append_bitexact()
        ref, _ = r.check_float(scores=True)
        _topc_checks(w, r, ref)
        st = r.last["state"]
        if c in (9, 10):   # the kept last block before the cut, clamped to time 0
            assert any(e.region == 1 and e.tau == 0 for e in st.kept[:st.n_kept])
    r.close()


@pytest.mark.parametrize("C", [2, 50])
def test_topc_small_candidate_sets(C):
    # 3-token frames: 3 to 45 candidates, so several of the top-C cluster's
    # eight slices are empty or hold a few keys, and C falls below and above
    # the candidate count
    w = W["infinity_rope"].replace(heads=1, head_dim=64, grid_h=1, grid_w=3, chunks=10, cut_chunks=(6,),
                                   topc=C)
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p, cut, scores=True)
        ref, _ = r.check_float(scores=True)
        _topc_checks(w, r, ref)
    r.close()


def test_inplace_rerotation_bitexact():
    # Sliding with a sink time shift: the sink is re-rotated in place by delta.
    w = W["tiny"].replace(heads=2, head_dim=128, grid_h=4, grid_w=8, sink_frames=2, chunks=6)
    r = Runner(w)
    for c in range(4):
        r.step(c, 0)
    kc, _ = r.cache.cache_views(0)
    F = w.frame_seqlen
    before = bits_of(kc[:, 0:2 * F]).copy()
    r.cache.reindex(5, B.RC_REINDEX_SINK)
    r.oracle.reindex(4, 5)
    r.step(4, 0)
    kc, _ = r.cache.cache_views(0)   # (a copy: the ring keeps 64-dim planes)
    after = bits_of(kc[:, 0:2 * F])
    want = rope_fp32_delta(before.transpose(1, 0, 2), 5, r.tables, r.pairs).transpose(1, 0, 2)
    assert np.array_equal(after, want)
    r.check_float()
    r.step(5, 0)
    r.check_float()
    r.close()


def test_deep_forcing_small():
    """Deep Forcing (rCM guide, strategy 4) on a small stream, every step: the
    region's tokens (chosen on the device from the kernel's own scores) equal
    the host top-C of those same scores bit for bit, region keys equal a CPU
    restatement of RoPE from their raw keys at the region's time, O / LSE
    within the float bar of fp64 and scores within SCORE_TOL of fp64."""
    w = W["deep_forcing"].replace(heads=2, grid_h=8, grid_w=8, chunks=14, df_budget_tokens=4 * 64)
    r = Runner(w)
    compacted = 0
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p, scores=True)
        r.check_append_bitexact()
        r.check_df_region_bitexact()
        ref, _ = r.check_float(scores=True)
        sg, sr = r.last["scores"], ref["scores"]
        assert len(sg) == len(sr)
        if len(sr):
            assert np.max(np.abs(sg - sr)) <= SCORE_TOL * max(1.0, np.max(np.abs(sr)))
        compacted += r.oracle.df.last_selection is not None
    assert compacted >= 8
    # every compaction's region also checked against the region fp64 scores choose
    assert r.df_fp64_checked == compacted
    r.close()


def test_deep_forcing_repeat_passes_and_zero_budget():
    # the selection of a chunk is made from the last pass before it
    w = W["deep_forcing"].replace(heads=2, grid_h=4, grid_w=8, chunks=9, passes=2,
                                  df_budget_tokens=2 * 32)
    r = Runner(w)
    compacted = 0
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p)
        r.check_df_region_bitexact()
        # fp64 scores of the last pass: the next chunk's region is checked against them
        r.check_float(scores=p == w.passes - 1)
        compacted += p == 0 and r.oracle.df.last_selection is not None
    assert compacted >= 3 and r.df_fp64_checked == compacted
    r.close()
    w0 = w.replace(df_budget_tokens=0, passes=1)
    r = Runner(w0)
    for c, p, g0, cut in rc_synth.stream_schedule(w0):
        r.step(c, p)
        assert r.last["state"].comp_tokens == 0
        r.check_float()
    r.close()


def test_relax_forcing_small():
    """Relax Forcing (rCM guide, strategy 5) on a small stream, every step:
    device pool scores within 1e-4 of fp64, the device selection = top-K of
    its own scores, region frames bit-exact copies of their keys at their own
    times, O / LSE within the float bar."""
    w = W["relax_forcing"].replace(heads=2, grid_h=8, grid_w=8, chunks=16, rf_history_frames=4)
    r = Runner(w)
    selected = 0
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p)
        r.check_append_bitexact()
        r.check_df_region_bitexact()
        r.check_float()
        selected += r.oracle.rf.last_scores is not None
    assert selected >= 8
    r.close()


@pytest.mark.parametrize("weight", [0.0, 1.0])
def test_relax_forcing_weights_passes_zero_history(weight):
    w = W["relax_forcing"].replace(heads=2, grid_h=4, grid_w=8, chunks=12, passes=2,
                                   rf_history_frames=3, rf_weight=weight)
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p)
        r.check_df_region_bitexact()
        r.check_float()
    r.close()
    w0 = w.replace(rf_history_frames=0, passes=1)
    r = Runner(w0)
    for c, p, g0, cut in rc_synth.stream_schedule(w0):
        r.step(c, p)
        assert r.last["state"].comp_tokens == 0
        r.check_float()
    r.close()


@pytest.mark.parametrize("alphas", [(0.9, 0.5), (0.0, 1.0)])
def test_memrope_small(alphas):
    """MemRoPE (rCM guide, MemRoPE tip) on a small stream, every step: memory
    frames bit-exact against the fp32 restatement of the device EMA with keys
    rotated to their times, O / LSE within the float bar of the fp64 oracle
    (which folds in fp64)."""
    w = W["memrope"].replace(heads=2, grid_h=8, grid_w=8, chunks=14, window_frames=6,
                             mr_alpha_long=alphas[0], mr_alpha_short=alphas[1])
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        r.step(c, p)
        r.check_append_bitexact()
        r.check_mem_bitexact()
        r.check_float()
    assert r.mem_folded >= 20
    r.close()


# ----------------------------------------------------------- full sizes
SAMPLE_ROWS = np.array([0, 1, 127, 128, 1559, 1560, 1561, 3119, 3120, 4607, 4608, 4679])


def _sampled(w, steps, layer=0, layers=None, scores_at=(), fp64_scores_at=()):
    """Drive a full-size stream through chunk max(steps). At ``steps``: the
    append bit-exact (first pass) and O / LSE on sampled rows against fp64.
    At ``scores_at``: the token scores positive with total mass below H Nq,
    and top-C exact on the kernel's own scores. At ``fp64_scores_at``: O /
    LSE on every row and head, every token score against fp64 within
    SCORE_TOL, and the top-C against the fp64 selection up to near-ties.
    Other chunks run without guard checks, integer state still exact."""
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([SAMPLE_ROWS, rng.integers(0, w.query_tokens, 20)]))
    r = Runner(w, layer=layer, layers=layers)
    last_chunk = max(steps)
    fp64_checked = 0
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        if c > last_chunk:
            break
        full = c in fp64_scores_at
        want_scores = c in scores_at or full
        r.step(c, p, cut, scores=want_scores, check=c in steps or want_scores)
        if c in steps:
            if p == 0:
                r.check_append_bitexact()
            if not full:
                r.check_float(rows=rows)
            st = r.last["state"]
            assert st.valid_tokens == min(g0 + 3, w.footprint_frames) * w.frame_seqlen or \
                w.policy == rc_synth.POLICY_INFINITY_ROPE
        if full:
            ref, _ = r.check_float(scores=True)
            _topc_checks(w, r, ref)
            fp64_checked += 1
        elif want_scores:
            sg = r.last["scores"]
            want = top_c(sg, np.arange(len(sg)) + 0, w.topc)  # positions; remapped below
            cand_lpos = np.nonzero(np.repeat([e.region == 1 for e in r.last["state"].kept[:r.last["state"].n_kept]],
                                             w.frame_seqlen))[0]
            assert np.array_equal(r.last["topc"], np.sort(cand_lpos[want]))
            assert np.all(sg > 0) and sg.sum() < w.heads * w.query_tokens
    assert fp64_checked == len(set(fp64_scores_at))
    r.close()


def test_full_wan13b_sampled():
    w = W["wan13b"]
    _sampled(w, steps={0, 1, 5, 6, 7}, layer=29, layers=30)


def test_full_large_sampled():
    _sampled(W["large"], steps={0, 1, 5, 6, 7})


def test_full_rolling_sink_sampled():
    # through the first roll period (block 12: the bank reversed) and into the
    # second (blocks 18, 19: the bank forward again, content period 12)
    _sampled(W["rolling_sink"], steps={0, 5, 6, 7, 8, 12, 18, 19})


def test_full_infinity_rope_sampled():
    """The Infinity-RoPE workload as configured (flush + cut 21 at chunks 27
    and 60 of the stream): sampled rows around both cuts, token scores and
    top-C (C = 4680) against fp64 at a steady-state chunk (10: 23400
    candidates) and right after the first cut (28: 9360 candidates)."""
    w = W["infinity_rope"]
    assert w.cut_chunks == (27, 60)
    _sampled(w, steps={0, 6, 7, 9, 10, 26, 27, 28, 60, 61}, scores_at={7, 9, 27, 60},
             fp64_scores_at={10, 28})


def test_full_deep_forcing_sampled():
    """Full-size Deep Forcing stream (12 heads, 1560-token frames, 3-frame
    deep sink + 18720-token region + 6-frame tail): the region selection
    exact every step, region keys bit-exact, sampled rows within the bar; at
    the steady-state chunk 8 every token score against fp64, and chunk 9's
    compaction (pool of 23400 tokens, budget 18720) against the region the
    fp64 scores choose, up to near-ties."""
    w = W["deep_forcing"]
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([SAMPLE_ROWS, rng.integers(0, w.query_tokens, 20)]))
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        if c > 9:
            break
        r.step(c, p, check=c in (0, 3, 4, 8, 9))
        if c in (0, 3, 4, 9):
            r.check_append_bitexact()
            r.check_df_region_bitexact()
            r.check_float(rows=rows)
        if c == 8:
            r.check_append_bitexact()
            r.check_df_region_bitexact()
            ref, _ = r.check_float(scores=True)
            sg, sr = r.last["scores"], ref["scores"]
            assert len(sg) == len(sr) == w.df_budget_tokens + 3 * w.frame_seqlen
            assert np.max(np.abs(sg - sr)) <= SCORE_TOL * max(1.0, np.max(np.abs(sr)))
    assert r.df_fp64_checked == 1
    st = r.last["state"]
    assert st.comp_tokens == w.df_budget_tokens and st.valid_tokens == w.footprint_tokens
    r.close()


def test_full_relax_forcing_sampled():
    """Full-size Relax Forcing stream (12 heads, 1560-token frames, sink 3 +
    12 history frames + tail 6): selection checks every step, region frames
    bit-exact and sampled rows within the bar at a few steps."""
    w = W["relax_forcing"]
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([SAMPLE_ROWS, rng.integers(0, w.query_tokens, 20)]))
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        if c > 9:
            break
        r.step(c, p)
        if c in (0, 3, 8, 9):
            r.check_append_bitexact()
            r.check_df_region_bitexact()
            r.check_float(rows=rows)
    r.close()



def test_full_memrope_sampled():
    """Full-size MemRoPE stream (12 heads, 1560-token frames, sink 3 + 2 memory
    frames + window 16): memory frames bit-exact every checked step."""
    w = W["memrope"]
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([SAMPLE_ROWS, rng.integers(0, w.query_tokens, 20)]))
    r = Runner(w)
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        if c > 9:
            break
        r.step(c, p)
        if c in (0, 6, 7, 9):
            r.check_append_bitexact()
            r.check_mem_bitexact()
            r.check_float(rows=rows)
    r.close()
