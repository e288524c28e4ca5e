"""Top-C over candidate sets that stretch the kernel's key storage.

The top-C kernel (K6b) runs as one cluster of 8 CTAs, each owning a
contiguous slice of the candidates; a slice's order keys stay in shared
memory for up to 45056 candidates (360448 in all) and are read back from the
logical-order scores in global memory beyond that. The full-size parity
streams stay far below either limit (Infinity-RoPE at 1560-token frames has
23400 candidates), so two streams with 64 x 64-token frames reach them:
  - Infinity-RoPE, one head: 15 history frames x 4096 = 61440 candidates,
    eight slices of 7680 in shared memory;
  - a sliding window of 93 frames, one head: 89 history frames x 4096 =
    364544 candidates, keys read from global memory.
The check is the one the selection has to meet exactly (rCM guide, strategy
4: keep the C highest-scoring tokens of the candidate range, ties to the
older token): the device's top-C equals the oracle's top_c on the device's
own scores, bit for bit, on steady-state chunks.
"""
import numpy as np
import pytest
import torch

import rc_synth
from oracle import top_c
from rolling_kv_cache_b200.cache import RollingKVCache

from gpu_util import dev_bf16
from rcutil import config_for

pytestmark = pytest.mark.gpu

CASES = {
    "slices_in_shared_memory": (
        rc_synth.WORKLOADS["infinity_rope"].replace(heads=1, head_dim=64, grid_h=64, grid_w=64, chunks=8,
                                                    cut_chunks=(), topc=20000), 49152),
    "keys_from_global_memory": (
        rc_synth.WORKLOADS["wan13b"].replace(layers=1, heads=1, head_dim=64, grid_h=64, grid_w=64,
                                             sink_frames=1, window_frames=92, chunks=33, passes=1,
                                             topc=20000), 360448),
}


@pytest.mark.parametrize("case", list(CASES))
def test_topc_large_candidate_sets(case):
    w, at_least = CASES[case]
    F = w.frame_seqlen
    cache = RollingKVCache(config_for(w))
    n_max = w.footprint_tokens
    C = w.topc
    checked = 0
    for c, p, g0, cut in rc_synth.stream_schedule(w):
        q, k, v = (dev_bf16(x) for x in rc_synth.chunk_qkv(w, 0, c, p))
        s = torch.zeros(n_max, dtype=torch.float32, device="cuda")
        t = torch.empty(C, dtype=torch.int32, device="cuda")
        cache.step(0, q, k, v, g0, scores=s, topc=t, C=C)
        torch.cuda.synchronize()
        cache.device_status()
        st = cache.state(0)
        n = st.n_candidates
        if n <= at_least:
            continue
        cand = []
        for li, e in enumerate(st.kept[:st.n_kept]):
            if e.region == 1:
                cand.extend(range(li * F, li * F + F))
        cand = np.array(cand)
        assert len(cand) == n
        scores = s[:n].cpu().numpy()
        sel = t.cpu().numpy()
        expect = top_c(scores, cand, C)
        m = min(C, n)
        assert np.array_equal(sel[:m], expect[:m])
        assert (sel[m:] == -1).all()
        checked += 1
    cache.close()
    assert checked >= 1
