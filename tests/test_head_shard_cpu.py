"""Head sharding on CPU: the head partition and the one exchange step.

Two gloo ranks each score the candidate tokens with their own head range
(fp64 oracle: per-head softmax probabilities summed over queries), sum the
vectors with an all-reduce, and select top-C from the sum; the result must be
the unsharded selection over all heads (a token's score is a plain sum over
heads, so the split changes nothing but the order of addition).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from rolling_kv_cache_b200.shard import head_ranges  # noqa: E402


@pytest.mark.parametrize("heads,world", [(12, 1), (12, 2), (12, 5), (12, 8), (40, 8), (3, 4), (0, 2)])
def test_head_ranges_cover_balanced_contiguous(heads, world):
    rs = head_ranges(heads, world)
    assert len(rs) == world
    assert rs[0][0] == 0 and rs[-1][1] == heads
    for (a0, a1), (b0, b1) in zip(rs, rs[1:]):
        assert a1 == b0
    sizes = [h1 - h0 for h0, h1 in rs]
    assert max(sizes) - min(sizes) <= 1
    assert sizes == sorted(sizes, reverse=True)


def test_head_ranges_rejects_bad_args():
    with pytest.raises(ValueError):
        head_ranges(4, 0)
    with pytest.raises(ValueError):
        head_ranges(-1, 2)


def _problem(seed=3, H=5, nq=24, nk=40, d=16):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((nq, H, d))
    k = rng.standard_normal((nk, H, d))
    v = rng.standard_normal((nk, H, d))
    vis = np.ones((nq, nk), dtype=bool)
    vis[:, 32:] = np.tril(np.ones((nq, 8), dtype=bool), k=-16)[:, :8]  # a masked current block
    cand = np.arange(4, 32)          # history tokens (sink = 0..3, current = 32..39)
    return q, k, v, vis, cand


def _scores(heads, q, k, v, vis, cand):
    from oracle.attention import column_scores, masked_sdpa
    s = np.zeros(len(cand))
    for h in heads:
        _, _, p = masked_sdpa(q[:, h], k[:, h], v[:, h], vis)
        s += column_scores([p], cand)
    return s


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from oracle import top_c
    from rolling_kv_cache_b200.shard import head_ranges
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, vis, cand = _problem()
        h0, h1 = head_ranges(q.shape[1], world)[rank]
        local = torch.from_numpy(_scores(range(h0, h1), q, k, v, vis, cand))
        dist.all_reduce(local, op=dist.ReduceOp.SUM)
        total = local.numpy()
        out_q.put((rank, total.tolist(), top_c(total, cand, 10).tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_score_allreduce_equals_unsharded():
    from oracle import top_c
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out_q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(out_q.get(timeout=10) for _ in range(2))
    q, k, v, vis, cand = _problem()
    full = _scores(range(q.shape[1]), q, k, v, vis, cand)
    want = top_c(full, cand, 10)
    for rank, total, sel in res:
        np.testing.assert_allclose(np.array(total), full, rtol=1e-12, atol=1e-12)
        assert sel == want.tolist()
    # every query row's probabilities sum to 1, so all heads together give
    # H x (rows) of mass over the visible keys; the candidates get part of it
    assert full.sum() <= q.shape[1] * q.shape[0] + 1e-9


def _state_rank_main(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    import rc_synth
    from rolling_kv_cache_b200 import binding as B
    from rolling_kv_cache_b200.cache import RollingKVCache
    from rolling_kv_cache_b200.shard import head_ranges
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = rc_synth.WORKLOADS["infinity_rope"]
        h0, h1 = head_ranges(w.heads, world)[rank]
        cache = RollingKVCache(bench.make_cfg(w, layers=1, heads=h1 - h0), device=None)
        trace = []
        for c in range(32):
            if c in w.cut_chunks:
                cache.reindex(w.cut_delta, B.RC_REINDEX_FLUSH | B.RC_REINDEX_CUT)
            cache.step(0, None, None, None, c * w.chunk_frames)
            st = cache.state(0)
            trace.append((st.n_candidates, st.valid_tokens,
                          tuple((e.content, e.tau, e.region) for e in st.kept[:st.n_kept])))
        gathered = [None] * world
        dist.all_gather_object(gathered, trace)
        out_q.put((rank, h1 - h0, all(t == gathered[0] for t in gathered), len(trace)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_compute_identical_integer_state():
    """Each rank plans its own head range; the plans (kept frames, time
    indices, candidates) agree with no exchange, so top-C indices agree."""
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_state_rank_main, args=(r, 2, port, out_q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(out_q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [6, 6]
    assert all(r[2] for r in res) and all(r[3] == 32 for r in res)


def _ulysses_main(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from rolling_kv_cache_b200.shard import head_ranges, heads_to_seq, seq_to_heads, token_ranges
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ok = []
        for N, H, d in [(12, 4, 3), (13, 5, 2), (7, 3, 4)]:      # uneven tokens and heads
            g = torch.Generator().manual_seed(N * 100 + H)
            x = torch.randn(N, H, d, generator=g)                  # the whole chunk, same on every rank
            t0, t1 = token_ranges(N, world)[rank]
            h0, h1 = head_ranges(H, world)[rank]
            xh = seq_to_heads(x[t0:t1].clone(), H)
            ok.append(torch.equal(xh, x[:, h0:h1]))
            back = heads_to_seq(xh * 2.0, H, t1 - t0)               # a per-head op, then back
            ok.append(torch.equal(back, 2.0 * x[t0:t1]))
        out_q.put((rank, ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ulysses_swaps_round_trip(world):
    """seq_to_heads gives each rank every token of its head range; heads_to_seq
    returns a per-head result to the token owners (uneven splits included)."""
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ulysses_main, args=(r, world, port, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [out_q.get(timeout=10) for _ in range(world)]
    assert all(all(ok) for _, ok in res)
