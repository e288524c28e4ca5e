"""Several caches in one process: two host threads driving two caches on one
GPU at once, and (where the box has two GPUs) a call made with the wrong
device current.

The launchers keep per-device, thread-safe lookups (kernel attributes, SM
counts, resident blocks per kernel), and every error message is per thread,
so two threads each driving their own cache on their own stream must get
exactly the bytes a single thread gets. The stream-K attention path (more
(head, query-block) units than SMs, partial rows merged by the combine
kernel) is the one exercised.
"""
import threading

import numpy as np
import pytest
import torch

import rc_synth
from rolling_kv_cache_b200 import binding as B
from rolling_kv_cache_b200.cache import RollingKVCache

from gpu_util import bits_of, dev_bf16
from rcutil import config_for

pytestmark = pytest.mark.gpu

# 64 heads x 3 query blocks = 192 units > 148 SMs; 240-token frames keep tiles ragged
W = rc_synth.Workload(name="threads", workload_id=14, layers=2, heads=64, head_dim=128, grid_h=12,
                      grid_w=20, chunk_frames=3, sink_frames=1, window_frames=6,
                      policy=rc_synth.POLICY_SLIDING, chunks=5, dist="normal_frame_mean")


def _stream(seed):
    cache = RollingKVCache(config_for(W))
    outs = []
    for c in range(W.chunks):
        for layer in range(W.layers):
            q, k, v = (dev_bf16(x) for x in rc_synth.chunk_qkv(W, layer, c, 0, seed))
            outs.append(bits_of(cache.step(layer, q, k, v, c * W.chunk_frames)))
    cache.device_status()
    cache.close()
    return outs


def test_two_threads_two_caches_match_sequential():
    want = {seed: _stream(seed) for seed in (1, 2)}
    got, errors = {}, []

    def worker(seed):
        try:
            with torch.cuda.stream(torch.cuda.Stream()):
                got[seed] = _stream(seed)
        except Exception as e:  # reported by the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(seed,)) for seed in (1, 2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=600)
    assert not errors, errors
    for seed in (1, 2):
        assert len(got[seed]) == len(want[seed])
        for a, b in zip(got[seed], want[seed]):
            assert np.array_equal(a, b)


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_call_with_another_device_current_is_rejected():
    w = rc_synth.WORKLOADS["tiny"]
    with torch.cuda.device(0):
        cache = RollingKVCache(config_for(w), torch.device("cuda", 0))
        q, k, v = (dev_bf16(x) for x in rc_synth.chunk_qkv(w, 0, 0, 0))
    with torch.cuda.device(1):
        out = torch.empty(q.shape, dtype=q.dtype, device="cuda:0")
        with pytest.raises(B.RcError) as e:
            B.rc_step(cache.handle, 0, q.data_ptr(), k.data_ptr(), v.data_ptr(), 0, 3, w.policy,
                      out.data_ptr())
        assert e.value.status == B.RC_EINVAL and "device" in str(e.value)
    assert cache.state(0).frames_committed == 0     # nothing was planned or enqueued
    with torch.cuda.device(0):
        cache.step(0, q, k, v, 0)
        torch.cuda.synchronize()
        cache.device_status()
    cache.close()
