"""rc_step_noalloc: the step for callers that cannot allocate device memory.

Its per-call scratch lives in the library's static device array instead of
the caller's block. It is checked here, through the C ABI, against rc_step on
an identical second cache fed identical inputs, for consecutive calls of a
stream that uses every scratch region (rotated queries, log-sum-exps, token
scores and top-C); at full size, where its attention grid has more
(head, query-block) units than the GPU has SMs, against the fp64 oracle.
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import rc_synth
from oracle import OracleStream, top_c
from rolling_kv_cache_b200 import binding as B
from rolling_kv_cache_b200.cache import RollingKVCache

from gpu_util import TOL_LSE, TOL_MAX, TOL_MEAN, bits_of, dev_bf16, f32
from rcutil import config_for, lib_kept, oracle_kept

pytestmark = pytest.mark.gpu


def _run(cache, fn, w, chunk, cut):
    if cut:
        cache.reindex(w.cut_delta, B.RC_REINDEX_FLUSH | B.RC_REINDEX_CUT)
    q, k, v = (dev_bf16(x) for x in rc_synth.chunk_qkv(w, 0, chunk, 0))
    out = torch.empty_like(q)
    lse = torch.empty((w.heads, q.shape[0]), dtype=torch.float32, device="cuda")
    sc = torch.zeros((w.footprint_tokens,), dtype=torch.float32, device="cuda")
    tc = torch.full((w.topc,), -7, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    fn(cache.handle, 0, q.data_ptr(), k.data_ptr(), v.data_ptr(), chunk * w.chunk_frames,
       w.chunk_frames, w.policy, out.data_ptr(), lse.data_ptr(), sc.data_ptr(), tc.data_ptr(),
       w.topc, stream)
    torch.cuda.synchronize()
    cache.device_status()
    n = cache.state(0).n_candidates
    return bits_of(out), lse.cpu().numpy(), sc.cpu().numpy()[:n], tc.cpu().numpy()


def test_noalloc_matches_rc_step_on_consecutive_calls():
    w = rc_synth.WORKLOADS["infinity_rope"].replace(heads=4, grid_h=20, grid_w=26, chunks=10,
                                                     cut_chunks=(8,), topc=1000)
    ref = RollingKVCache(config_for(w))
    alt = RollingKVCache(config_for(w))
    compared = 0
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        o1, l1, s1, t1 = _run(ref, B.rc_step, w, c, cut)
        o2, l2, s2, t2 = _run(alt, B.rc_step_noalloc, w, c, cut)
        err = np.abs(f32(o1).astype(np.float64) - f32(o2))
        assert err.max() <= 2e-2 and err.mean() <= 2e-3
        assert np.abs(l1 - l2).max() <= 1e-2
        assert len(s1) == len(s2)
        if len(s1):
            assert np.abs(s1 - s2).max() <= 1e-3 * max(1.0, np.abs(s1).max())
            # the selection is exact on each call's own scores
            st = alt.state(0)
            lpos = np.nonzero(np.repeat([e.region == 1 for e in st.kept[:st.n_kept]], w.frame_seqlen))[0]
            want = np.sort(lpos[top_c(s2, np.arange(len(s2)), w.topc)])
            n = min(w.topc, len(s2))
            assert np.array_equal(t2[:n], want) and np.all(t2[n:] == -1)
            # against rc_step's selection: differences only among near-ties of
            # the C-th score (the two runs accumulate scores in different orders)
            if n < len(s1):
                kth = np.sort(s1)[::-1][n - 1]
                where = {int(x): i for i, x in enumerate(lpos)}
                for x in set(t1[:n].tolist()) ^ set(t2[:n].tolist()):
                    assert abs(s1[where[x]] - kth) <= 1e-3 * max(1.0, kth)
            else:
                assert np.array_equal(t1, t2)
            compared += 1
    assert compared >= 2
    ref.close()
    alt.close()


def test_noalloc_rejects_scratch_beyond_its_maximum():
    w = rc_synth.WORKLOADS["large"]   # 40 heads x 4680 queries: 48 MB of rotated queries
    cache = RollingKVCache(config_for(w, window_frames=3, sink_frames=0))
    q = torch.zeros((w.query_tokens, w.heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(B.RcError) as e:
        B.rc_step_noalloc(cache.handle, 0, q.data_ptr(), q.data_ptr(), q.data_ptr(), 0, 3, w.policy,
                          out.data_ptr())
    assert e.value.status == B.RC_ERANGE and "static maximum" in str(e.value)
    assert cache.state(0).frames_committed == 0     # nothing happened
    cache.close()


def test_noalloc_full_size_grid_beyond_sms_against_oracle():
    # The Infinity-RoPE workload at full size: 12 heads x 128, 4680-query
    # chunks, 32760 cached tokens, token scores + top-C 4680 every step. Its
    # step scratch (14.9 MB) fits the static array, and its 12 x 19 = 228
    # (head, query-block) units exceed the SM count, so the one-CTA-per-unit
    # grid runs in more than one wave.
    w = rc_synth.WORKLOADS["infinity_rope"].replace(chunks=9)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert w.heads * ((w.query_tokens + 255) // 256) > sms
    cache = RollingKVCache(config_for(w))
    oracle = OracleStream(w)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 255, 256, 1559, 1560, 3119, 3120, 4607, 4679],
                                     rng.integers(0, w.query_tokens, 22)]))
    checked = 0
    for c in range(w.chunks):
        o, lse, sc, tc = _run(cache, B.rc_step_noalloc, w, c, False)
        kept = oracle.step(c, 0)
        st = cache.state(0)
        assert lib_kept(st) == oracle_kept(kept)
        # top-C exact on the call's own scores (ties to the lower index)
        lpos = np.nonzero(np.repeat([e.region == 1 for e in st.kept[:st.n_kept]], w.frame_seqlen))[0]
        n = min(w.topc, len(sc))
        if n:
            assert np.array_equal(tc[:n], np.sort(lpos[top_c(sc, np.arange(len(sc)), w.topc)]))
        assert np.all(tc[n:] == -1)
        if c in (0, 7, 8):
            ref = oracle.outputs(rows=rows)
            err = np.abs(f32(o)[rows].astype(np.float64) - ref["o"])
            lerr = np.abs(lse[:, rows] - ref["lse"])
            assert err.max() <= TOL_MAX and err.mean() <= TOL_MEAN and lerr.max() <= TOL_LSE, \
                (c, err.max(), err.mean(), lerr.max())
            checked += 1
    assert checked == 3
    cache.close()
