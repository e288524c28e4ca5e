"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, weak scaling.

Each rank runs its own independent stream (here: host-only caches, so the
library's integer engine runs on every rank with no GPU); the whole-job
figures are the summed work over the slowest rank's time. No collective sits
on the data path: ranks only meet for the barrier and the two reductions.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    import rc_synth
    from rolling_kv_cache_b200 import binding as B
    from rolling_kv_cache_b200.cache import RollingKVCache
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # each rank: its own stream of the wan13b schedule through the engine
        w = rc_synth.WORKLOADS["wan13b"]
        cache = RollingKVCache(bench.make_cfg(w, layers=2), device=None)
        steps = 4 + rank   # unequal work per rank
        for c in range(steps):
            for p in range(w.passes):
                for l in range(2):
                    cache.step(l, None, None, None, c * 3)
        st = cache.state(1)
        dist.barrier()
        ms, work = bench.aggregate_over_ranks(10.0 * (rank + 1), float(steps))
        q.put((rank, ms, work, st.frames_committed, st.valid_tokens))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, work, frames, valid in res:
        assert ms == 20.0                 # slowest rank
        assert work == 4.0 + 5.0          # summed over ranks
    assert res[0][3] == 12 and res[1][3] == 15   # independent streams
    assert res[0][4] == 12 * 1560 and res[1][4] == 15 * 1560


def test_single_process_aggregate_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_over_ranks(3.5, 7.0) == (3.5, 7.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    import rc_synth
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 0, 2
    assert bench.run_reference(A, rc_synth.WORKLOADS["wan13b"]) == 0
    assert capsys.readouterr().out == ""
