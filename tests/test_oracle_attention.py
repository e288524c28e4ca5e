"""Pins for the oracle's attention, scores and top-C."""
import math

import numpy as np
import pytest

import rc_synth
from oracle import (OracleStream, column_scores, masked_sdpa, rope_angles, rope_apply,
                    top_c, visibility)

import pins


def test_sdpa_matches_torch():
    pins.check_sdpa_vs_torch(masked_sdpa)


def test_visibility_definition():
    qr = np.array([0, 0, 1, 2, 2])
    kr = np.array([-1, -1, 0, 1, 2, 0])
    for m in (1, 3):
        vis = visibility(qr, kr, m)
        for i in range(len(qr)):
            for j in range(len(kr)):
                want = kr[j] == -1 or (kr[j] // m) <= (qr[i] // m)
                assert vis[i, j] == want


def test_softmax_invariants():
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((6, 16)), rng.standard_normal((20, 16)), rng.standard_normal((20, 16))
    vis = rng.random((6, 20)) < 0.5
    vis[:, 3] = True
    o, lse, p = masked_sdpa(q, k, v, vis)
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(p[~vis] == 0)
    # one visible key -> output is that key's value
    one = np.zeros_like(vis)
    one[:, 7] = True
    o1, _, _ = masked_sdpa(q, k, v, one)
    assert np.allclose(o1, v[7][None], atol=1e-14)
    # q = 0 -> uniform weights: mean of visible values, lse = log(count)
    o0, l0, _ = masked_sdpa(0 * q, k, v, vis)
    for i in range(6):
        assert np.allclose(o0[i], v[vis[i]].mean(axis=0), atol=1e-13)
        assert abs(l0[i] - math.log(vis[i].sum())) < 1e-13


def test_uniform_time_shift_leaves_scores_unchanged():
    rng = np.random.default_rng(7)
    n = 40
    q = rng.standard_normal((n, 1, 128))
    k = rng.standard_normal((n, 1, 128))
    t = rng.integers(0, 50, n)
    h, w = rng.integers(0, 30, n), rng.integers(0, 52, n)
    s0 = rope_apply(q, rope_angles(t, h, w, 128, 1e4))[:, 0] @ \
        rope_apply(k, rope_angles(t[::-1], h, w, 128, 1e4))[:, 0].T
    for c in (1, 17, 300):
        s1 = rope_apply(q, rope_angles(t + c, h, w, 128, 1e4))[:, 0] @ \
            rope_apply(k, rope_angles(t[::-1] + c, h, w, 128, 1e4))[:, 0].T
        assert np.max(np.abs(s1 - s0)) <= 1e-12 * max(1.0, np.max(np.abs(s0)))


def test_topc_bruteforce():
    pins.check_topc_bruteforce(top_c)


def test_column_scores_total_mass():
    rng = np.random.default_rng(9)
    ps = []
    for h in range(3):
        q, k, v = rng.standard_normal((5, 8)), rng.standard_normal((12, 8)), rng.standard_normal((12, 8))
        ps.append(masked_sdpa(q, k, v, np.ones((5, 12), bool))[2])
    total = column_scores(ps, np.arange(12)).sum()
    assert abs(total - 3 * 5) < 1e-12


def test_column_scores_are_the_logit_bias_gradient():
    pins.check_column_scores_autograd(column_scores)


TINY = rc_synth.Workload(name="brute", workload_id=9, layers=1, heads=2, head_dim=8,
                         grid_h=2, grid_w=2, chunk_frames=2, sink_frames=1,
                         window_frames=100, policy=rc_synth.POLICY_SLIDING, chunks=4)


@pytest.mark.parametrize("policy", [rc_synth.POLICY_SLIDING, rc_synth.POLICY_NONE])
@pytest.mark.parametrize("mask_block", [1, 2])
def test_window_covering_history_is_full_causal_attention(policy, mask_block):
    """P3: with the window >= the history the chunked step equals brute-force
    block-causal attention over the whole sequence (scalar loops, complex RoPE)."""
    w = TINY.replace(policy=policy, mask_block_frames=mask_block)
    st = OracleStream(w)
    F, B, d = w.frame_seqlen, w.chunk_frames, w.head_dim
    hh = [n // w.grid_w for n in range(F)]
    ww = [n % w.grid_w for n in range(F)]

    def frames_of(c, tid):
        return st.tensor(c, 0, tid)

    for c in range(w.chunks):
        st.step(c, 0)
        out = st.outputs()
        for h in range(w.heads):
            keys, vals, kframe = [], [], []
            for g in range(B * c + B):
                kc = frames_of(g // B, rc_synth.TENSOR_K)[(g % B) * F:(g % B + 1) * F]
                vc = frames_of(g // B, rc_synth.TENSOR_V)[(g % B) * F:(g % B + 1) * F]
                for n in range(F):
                    keys.append(pins.complex_rope(kc[n, h], g, hh[n], ww[n], d, w.theta))
                    vals.append(vc[n, h])
                    kframe.append(g)
            qc = frames_of(c, rc_synth.TENSOR_Q)
            qs, vis = [], []
            for n in range(B * F):
                g = B * c + n // F
                qs.append(pins.complex_rope(qc[n, h], g, hh[n % F], ww[n % F], d, w.theta))
                # block-causal: keys of earlier chunks always; this chunk's by block
                vis.append([kf < B * c or ((kf - B * c) // mask_block) <= ((g - B * c) // mask_block)
                            for kf in kframe])
            o_ref, lse_ref = pins.brute_attention(qs, keys, vals, vis)
            assert np.allclose(out["o"][:, h], o_ref, rtol=0, atol=1e-12)
            assert np.allclose(out["lse"][h], lse_ref, rtol=0, atol=1e-12)


def test_scores_and_topc_on_stream():
    w = rc_synth.Workload(name="sc", workload_id=10, layers=1, heads=2, head_dim=8, grid_h=2,
                          grid_w=2, chunk_frames=2, sink_frames=2, window_frames=6,
                          policy=rc_synth.POLICY_INFINITY_ROPE, chunks=6, ir_f_limit=6,
                          ir_sink_blocks=1, ir_cache_blocks=3, topc=5)
    st = OracleStream(w)
    for c in range(w.chunks):
        kept = st.step(c, 0)
        out = st.outputs(want_scores=True)
        n_hist = sum(k.region == "hist" for k in kept) * w.frame_seqlen
        assert len(out["scores"]) == n_hist
        if n_hist:
            # every candidate is visible to every query, so scores are sums of
            # probabilities: positive and at most heads * queries
            assert np.all(out["scores"] > 0)
            assert out["scores"].sum() < w.heads * w.query_tokens
            assert list(out["topc"]) == sorted(out["topc"])
            assert len(out["topc"]) == min(w.topc, n_hist)


def _bf16_round(x):
    a = np.asarray(x, dtype=np.float32)
    b = a.view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16   # round to nearest even
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("d", [128, 64])
def test_score_tolerance_covers_bf16_storage(d, monkeypatch):
    """The GPU parity bar for token scores (SCORE_TOL of the largest) against
    what storing the rotated queries and keys in bf16 alone does to the fp64
    scores on the score parity stream (Infinity-RoPE, two RoPE cuts): the
    bar must sit above that, with room for the fp32 arithmetic and the
    in-place re-rotations, and within a small factor of it."""
    import oracle.stream as stream_mod
    from rcutil import SCORE_TOL
    w = rc_synth.WORKLOADS["infinity_rope"].replace(heads=2, head_dim=d, grid_h=8, grid_w=8, chunks=18,
                                                   cut_chunks=(9, 13), topc=100)
    o = OracleStream(w)
    worst = 0.0
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        if cut:
            o.reindex(1 | 2, w.cut_delta)
        o.step(c, p)
        monkeypatch.setattr(stream_mod, "rope_apply", rope_apply)
        exact = o.outputs(want_scores=True)["scores"]
        monkeypatch.setattr(stream_mod, "rope_apply", lambda x, ang: _bf16_round(rope_apply(x, ang)))
        stored = o.outputs(want_scores=True)["scores"]
        if len(exact):
            worst = max(worst, np.max(np.abs(exact - stored)) / max(1.0, np.max(np.abs(exact))))
    assert worst > 0.0
    assert 1.5 * worst <= SCORE_TOL <= 8 * worst, (worst, SCORE_TOL)
