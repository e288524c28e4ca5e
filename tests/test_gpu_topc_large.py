"""Top-C over a candidate set too large for the kernel's shared-memory keys.

The top-C kernel (K6b) keeps the candidates' order keys in shared memory for
up to 49152 candidates and reads them back from the logical-order scores in
global memory beyond that. The full-size parity streams stay under the limit
(Infinity-RoPE at 1560-token frames has 23400 candidates), so this stream uses
64 x 64-token frames: 15 history frames x 4096 = 61440 candidates. The check
is the one the selection has to meet exactly (rCM guide, strategy 4: keep the
C highest-scoring tokens of the candidate range, ties to the older token): the
device's top-C equals the oracle's top_c on the device's own scores, bit for
bit, on a steady-state chunk.
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


def test_topc_above_shared_memory_keys():
    w = rc_synth.WORKLOADS["infinity_rope"].replace(heads=1, head_dim=64, grid_h=64, grid_w=64,
                                                    chunks=8, cut_chunks=(), topc=20000)
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
        if n <= 49152:
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
