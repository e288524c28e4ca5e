"""Head sharding of one stream, emulated on one GPU.

Under head sharding each rank's cache holds a contiguous range of the heads
and runs every step on that range only; the path needs no exchange except one
sum of the ranks' token-score vectors before top-C (heads are independent in
the RoPE, the append, the attention and the score pass). Here the two ranks'
caches live on one GPU and run one after the other (no rank waits on
another), so the sharded path is checked against the unsharded cache:
per-head outputs within the float tolerance, the summed scores within 1e-3
relative, and rc_select_topc on the sum bit-exact against the host selection
on the same sum, and up to near-ties against the unsharded top-C.
"""
import numpy as np
import pytest
import torch

import rc_synth
from oracle import top_c
from rolling_kv_cache_b200 import binding as B
from rolling_kv_cache_b200.cache import RollingKVCache

from gpu_util import dev_bf16
from rcutil import config_for
from rolling_kv_cache_b200.shard import head_ranges

pytestmark = pytest.mark.gpu


def test_head_sharded_matches_unsharded():
    w = rc_synth.WORKLOADS["infinity_rope"].replace(heads=5, grid_h=8, grid_w=8, chunks=12,
                                                    cut_chunks=(7,), topc=100)
    world = 2
    ranges = head_ranges(w.heads, world)
    full = RollingKVCache(config_for(w))
    shards = [RollingKVCache(config_for(w.replace(heads=h1 - h0))) for h0, h1 in ranges]
    n_max = w.footprint_tokens
    C = w.topc
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        if cut:
            for cache in [full] + shards:
                cache.reindex(w.cut_delta, B.RC_REINDEX_FLUSH | B.RC_REINDEX_CUT)
        q, k, v = (dev_bf16(x) for x in rc_synth.chunk_qkv(w, 0, c, p))
        s_full = torch.zeros(n_max, dtype=torch.float32, device="cuda")
        t_full = torch.empty(C, dtype=torch.int32, device="cuda")
        o_full = full.step(0, q, k, v, g0, scores=s_full, topc=t_full, C=C)
        s_sum = torch.zeros(n_max, dtype=torch.float32, device="cuda")
        for (h0, h1), cache in zip(ranges, shards):
            s_r = torch.zeros(n_max, dtype=torch.float32, device="cuda")
            o_r = cache.step(0, q[:, h0:h1].contiguous(), k[:, h0:h1].contiguous(),
                             v[:, h0:h1].contiguous(), g0, scores=s_r)
            torch.cuda.synchronize()
            diff = (o_r.float() - o_full[:, h0:h1].float()).abs()
            assert diff.max().item() <= 2e-2 and diff.mean().item() <= 2e-3
            s_sum += s_r            # the all-reduce of the score vectors
        t_sh = shards[0].select_topc(0, s_sum, C)
        torch.cuda.synchronize()
        full.device_status()
        for cache in shards:
            cache.device_status()
        st = full.state(0)
        n = st.n_candidates
        for cache in shards:      # every rank computes the same integer state
            assert cache.state(0).n_candidates == n
        if n == 0:
            assert (t_sh.cpu().numpy() == -1).all()
            continue
        a, b = s_full[:n].cpu().numpy(), s_sum[:n].cpu().numpy()
        assert np.abs(a - b).max() <= 1e-3 * max(1.0, float(a.max()))
        # candidates' logical indices: history tokens of the kept list, in order
        F = w.frame_seqlen
        cand = []
        for li, e in enumerate(st.kept[:st.n_kept]):
            if e.region == 1:
                cand.extend(range(li * F, li * F + F))
        cand = np.array(cand)
        assert len(cand) == n
        # exact on the kernel's own (summed) scores
        sel = t_sh.cpu().numpy()
        expect = top_c(b, cand, C)
        m = min(C, n)
        assert np.array_equal(sel[:m], expect[:m])
        assert (sel[m:] == -1).all()
        # against the unsharded selection: swaps only among near-ties of the C-th score
        only = set(t_full.cpu().numpy()[:m].tolist()) ^ set(sel[:m].tolist())
        if only and n > C:
            kth = np.sort(b)[::-1][C - 1]
            pos = {int(x): i for i, x in enumerate(cand)}
            for x in only:
                assert abs(b[pos[x]] - kth) <= 1e-3 * max(1.0, float(kth))
    for cache in [full] + shards:
        cache.close()
