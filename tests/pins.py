"""Independent checks that pin the fp64 oracle to the pages and to mathematics.

Each ``check_*`` function takes the oracle piece under test as an argument and
raises AssertionError on a mismatch, so the same check runs against the real
oracle (tests/test_oracle_*.py) and against copies of it with a plausible
mistake planted (tests/test_oracle_mutations.py), which it must reject.
Nothing here reuses the oracle's formulas: RoPE is recomputed with complex
numbers, attention with scalar Python loops, top-C by exhaustive search,
token scores as the gradient of the summed log-sum-exp (torch autograd).
"""
from __future__ import annotations

import cmath
import itertools
import math
import os
import re

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- fixtures
def load_rolling_sink_table():
    rows = {}
    with open(os.path.join(GOLDEN, "rolling_sink_k6_s5.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            step, rest = line.split(":")
            rows[int(step)] = [tuple(int(x) for x in e.split(",")) for e in rest.split()]
    return rows


def load_infinity_rope_table():
    rows = {}
    with open(os.path.join(GOLDEN, "infinity_rope_b3_f21_c6.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            chunk, rest = line.split(":", 1)
            parts = rest.split("|")
            assert len(parts) == 3
            rows[int(chunk)] = [
                [tuple(int(x) for x in e.split(":")) for e in p.split()] for p in parts]
    return rows


def load_lingbot_numbers():
    out = {}
    with open(os.path.join(GOLDEN, "lingbot_token_arithmetic.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split("=")
                out[k] = int(v)
    return out


# ------------------------------------------------------------------ policy
def check_rolling_sink(policy_cls, K=6, S=5, B=3):
    """Sink (block, time) per step equals the hand enumeration; recent/current too."""
    table = load_rolling_sink_table()
    pol = policy_cls(2, B, S * B, (K - S + 1) * B, rs_bank_blocks=K, rs_sink_blocks=S)
    last = max(table)
    for i in range(last + 1):
        kept = pol.step(i * B, B)
        if i not in table:
            continue
        sink = [k for k in kept if k.region == "sink"]
        hist = [k for k in kept if k.region == "hist"]
        cur = [k for k in kept if k.region == "cur"]
        got = []
        for j in range(0, len(sink), B):
            blk = sink[j:j + B]
            cb, tb = blk[0].content // B, blk[0].tau // B
            for o, e in enumerate(blk):
                assert e.content == cb * B + o and e.tau == tb * B + o, (i, e)
            got.append((cb, tb))
        assert got == table[i], (i, got, table[i])
        assert [(e.content, e.tau) for e in hist] == [((i - 1) * B + o, (i - 1) * B + o) for o in range(B)]
        assert [(e.content, e.tau, e.rank) for e in cur] == [(i * B + o, i * B + o, o) for o in range(B)]


def check_infinity_rope(policy_cls, chunks=100, cuts=(27, 60), delta=21):
    table = load_infinity_rope_table()
    pol = policy_cls(3, 3, 3, 18, ir_f_limit=21, ir_sink_blocks=1, ir_cache_blocks=6)
    for c in range(chunks):
        if c in cuts:
            pol.reindex(1 | 2, delta)
        kept = pol.step(3 * c, 3)
        if c not in table:
            continue
        want_sink, want_hist, want_cur = table[c]
        got = [[(k.content, k.tau) for k in kept if k.region == r] for r in ("sink", "hist", "cur")]
        assert got == [want_sink, want_hist, want_cur], (c, got)


def check_lingbot_numbers(policy_cls, frame_seqlen, sink_frames, window_frames, chunk_frames, chunks):
    nums = load_lingbot_numbers()
    assert nums["latent_h_px"] * nums["latent_w_px"] // nums["patch_area"] == nums["frame_seqlen"]
    assert frame_seqlen == nums["frame_seqlen"]
    assert (sink_frames + window_frames) * frame_seqlen == nums["cache_tokens"]
    assert sink_frames * frame_seqlen == nums["sink_tokens"]
    assert chunk_frames * frame_seqlen == nums["chunk_tokens"]
    pol = policy_cls(1, chunk_frames, sink_frames, window_frames)
    prev = []
    full = False
    for c in range(chunks):
        kept = pol.step(c * chunk_frames, chunk_frames)
        tokens = len(kept) * frame_seqlen
        assert tokens <= nums["cache_tokens"]
        if full:
            assert tokens == nums["cache_tokens"]
            gone = set(k.content for k in prev) - set(k.content for k in kept)
            assert len(gone) * frame_seqlen == nums["evicted_per_chunk"]
            assert all(g >= sink_frames for g in gone)
            assert [k.content for k in kept[:sink_frames]] == list(range(sink_frames))
        full = full or tokens == nums["cache_tokens"]
        prev = kept
    assert full


# -------------------------------------------------------------------- rope
def complex_rope(x, t, h, w, head_dim, theta):
    """RoPE by complex multiplication, written independently: x [d] -> [d]."""
    c = head_dim // 2
    p_hw = c // 3
    p_t = c - 2 * p_hw
    out = []
    for m in range(c):
        if m < p_t:
            pos, j, P = t, m, p_t
        elif m < p_t + p_hw:
            pos, j, P = h, m - p_t, p_hw
        else:
            pos, j, P = w, m - p_t - p_hw, p_hw
        freq = math.pow(theta, -j / P)
        z = complex(x[2 * m], x[2 * m + 1]) * cmath.exp(1j * pos * freq)
        out += [z.real, z.imag]
    return np.array(out)


def check_rope_complex(rope_angles_fn, rope_apply_fn, head_dim=128, theta=10000.0, seed=0):
    rng = np.random.default_rng(seed)
    n = 7
    x = rng.standard_normal((n, 2, head_dim))
    t = rng.integers(0, 400, n)
    h = rng.integers(0, 30, n)
    w = rng.integers(0, 52, n)
    got = rope_apply_fn(x, rope_angles_fn(t, h, w, head_dim, theta))
    for i in range(n):
        for hd in range(2):
            want = complex_rope(x[i, hd], t[i], h[i], w[i], head_dim, theta)
            assert np.allclose(got[i, hd], want, rtol=0, atol=1e-12), i


# --------------------------------------------------------------- attention
def brute_attention(q_rows, keys, values, visible):
    """Scalar-loop softmax attention: lists of vectors, visible[i][j] bool."""
    d = len(q_rows[0])
    outs, lses = [], []
    for i, q in enumerate(q_rows):
        s = []
        for j, k in enumerate(keys):
            if visible[i][j]:
                s.append((j, sum(a * b for a, b in zip(q, k)) / math.sqrt(d)))
        m = max(v for _, v in s)
        e = [(j, math.exp(v - m)) for j, v in s]
        z = sum(v for _, v in e)
        o = [sum(wt * values[j][c] for j, wt in e) / z for c in range(d)]
        outs.append(o)
        lses.append(m + math.log(z))
    return np.array(outs), np.array(lses)


def check_sdpa_vs_torch(masked_sdpa_fn, seed=0):
    import torch
    rng = np.random.default_rng(seed)
    for nq, nk, d in ((5, 9, 8), (33, 70, 64), (17, 130, 128)):
        q, k, v = (rng.standard_normal((n, d)) for n in (nq, nk, nk))
        vis = rng.random((nq, nk)) < 0.7
        vis[:, 0] = True
        o, lse, p = masked_sdpa_fn(q, k, v, vis)
        t = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
            attn_mask=torch.from_numpy(vis)[None])
        assert np.allclose(o, t[0].numpy(), rtol=0, atol=1e-12)
        s = (q @ k.T) / math.sqrt(d)
        ref_lse = torch.logsumexp(torch.from_numpy(np.where(vis, s, -np.inf)), dim=1).numpy()
        assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def check_topc_bruteforce(top_c_fn, seed=0):
    """The returned set is the unique C-subset in which every member beats
    every non-member under (higher score, then lower logical index)."""
    rng = np.random.default_rng(seed)
    for trial in range(40):
        n = int(rng.integers(1, 9))
        C = int(rng.integers(0, n + 1))
        scores = rng.integers(0, 4, n).astype(np.float64)  # many ties
        idx = np.sort(rng.choice(100, n, replace=False))
        got = list(top_c_fn(scores, idx, C))
        winners = []
        for sub in itertools.combinations(range(n), C):
            rest = [i for i in range(n) if i not in sub]
            if all((scores[a] > scores[b]) or (scores[a] == scores[b] and idx[a] < idx[b])
                   for a in sub for b in rest):
                winners.append(sorted(int(idx[a]) for a in sub))
        assert len(winners) == 1
        assert got == winners[0], (scores, idx, C, got, winners)


def check_column_scores_autograd(column_scores_fn, seed=0):
    """Token scores as a derivative: for lse_q = log sum_j exp(s_qj + b_j),
    d lse_q / d b_j is the probability p_qj, so the gradient of the summed
    log-sum-exp over every head and query with respect to a per-key logit
    bias b is each key's received attention mass. torch autograd computes it
    from the logits alone; the oracle's function gets the probabilities and a
    candidate subset of the key columns, whose scores it must return in the
    subset's order."""
    import torch
    rng = np.random.default_rng(seed)
    for H, nq, nk, d in ((1, 3, 5, 4), (3, 7, 19, 8), (4, 12, 40, 16)):
        q = torch.from_numpy(rng.standard_normal((H, nq, d)))
        k = torch.from_numpy(rng.standard_normal((H, nk, d)))
        vis = rng.random((nq, nk)) < 0.6
        vis[:, int(rng.integers(nk))] = True
        logits = torch.where(torch.from_numpy(vis)[None], q @ k.transpose(1, 2) / math.sqrt(d),
                             torch.tensor(-math.inf, dtype=torch.float64))
        b = torch.zeros(nk, dtype=torch.float64, requires_grad=True)
        torch.logsumexp(logits + b, dim=2).sum().backward()
        mass = b.grad.numpy()
        p_per_head = [torch.softmax(logits[h], dim=1).numpy() for h in range(H)]
        cols = np.sort(rng.choice(nk, size=max(1, nk // 2), replace=False))
        got = np.asarray(column_scores_fn(p_per_head, cols))
        assert got.shape == cols.shape, (got.shape, cols.shape)
        assert np.allclose(got, mass[cols], rtol=0, atol=1e-12), (got, mass[cols])
