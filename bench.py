#!/usr/bin/env python
"""Benchmark of the chunked attention step over the bounded KV cache.

Workload (default): the Wan2.1-1.3B-shaped sliding-window stream -- 30 layers,
12 heads x 128, 1560-token frames (30x52 latent grid), 3-frame chunks (4680
queries), sink 1 frame + window 18 frames (29640 cached tokens per head), 4
denoise passes + 1 clean cache-refresh pass per chunk. One bench step = one
chunk through all 30 layers x 5 passes = 150 rc_step calls (each: fused RoPE +
append, tcgen05 attention). Synthetic seeded inputs (N(0,1) + per-frame mean
N(0, 0.5), bf16); the cache is driven to steady state (full window) before
warm-up.

Prints one JSON line. ``value`` is chunk-attention TFLOP/s (algorithmic FLOPs
4*d*H*visible pairs over the timed region's device time, summed over ranks);
``frames_per_s_per_layer`` the streamed latent frame rate per layer.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (one head of one layer-pass per step) on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import rc_synth  # noqa: E402

METRIC = "chunk-attention TFLOP/s vs bf16 peak; streamed latent frames/s per layer"
UNIT = "TFLOP/s"


def visible_pairs(w, n_hist_frames: int) -> int:
    """(query, key) pairs the chunk attention computes (frame-causal in chunk)."""
    F, B, m = w.frame_seqlen, w.chunk_frames, w.mask_block_frames
    pairs = 0
    for r in range(B):
        vis = sum(1 for r2 in range(B) if r2 // m <= r // m)
        pairs += F * (n_hist_frames * F + vis * F)
    return pairs


def attention_flops(w, n_hist_frames: int, heads=None) -> float:
    return 4.0 * w.head_dim * (w.heads if heads is None else heads) * visible_pairs(w, n_hist_frames)


def steady_hist_frames(w) -> int:
    """Frames' worth of cached keys besides the chunk at steady state (the
    Deep Forcing region counts as budget / F frames)."""
    return w.footprint_tokens // w.frame_seqlen - w.chunk_frames


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("attn_fwd.cu", "attn_common.cuh", "ptx.cuh", "kernels.cuh"):
        with open(os.path.join(ROOT, "rolling_kv_cache_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def attention_traffic():
    """DRAM bytes per attention launch (dram__bytes_read.sum +
    dram__bytes_write.sum of one ncu capture of a steady-state layer-pass),
    from the machine-readable capture summary, if that capture was taken on
    the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "attention_wan13b_ncu.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    return float(rec["dram_bytes_per_launch"])


def _clock_fields(obj, path=""):
    """(key path, value) of every numeric field under a clock-like key."""
    if isinstance(obj, dict):
        out = []
        for k, v in obj.items():
            out += _clock_fields(v, f"{path}/{k}".lower())
        return out
    if isinstance(obj, (int, float)) and not isinstance(obj, bool) and ("mhz" in path or "clock" in path) \
            and "mem" not in path and "max" not in path and 300 <= obj <= 3000:
        return [(path, float(obj))]
    return []


def peak_clock_mhz(peaks, sustained: bool):
    """SM clock under which the measured GEMM peak was taken, if the peaks
    record it: among the clock fields, those naming (or not) the sustained
    run, preferring ones tied to the bf16 GEMM and to a median."""
    cands = [(pth, v) for pth, v in _clock_fields(peaks) if ("sustain" in pth) == sustained]
    if not cands:
        return None

    def rank(item):
        pth = item[0]
        return (-sum(w in pth for w in ("bf16", "gemm", "matmul", "mm", "tflops")), -("median" in pth), pth)
    return sorted(cands, key=rank)[0][1]


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.gpu_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return False
        time.sleep(0.3)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)
        return False

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in self.rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        loaded = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


def aggregate_over_ranks(ms: float, work: float, device=None):
    """(max of ms, sum of work) over the ranks of the default process group.

    Whole-job throughput = summed work over the slowest rank's time. With a
    single process it returns its inputs. Every rank calls it at the same
    point (same collectives, same order)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms, work
    t_max = torch.tensor([ms], dtype=torch.float64, device=device)
    t_sum = torch.tensor([work], dtype=torch.float64, device=device)
    dist.all_reduce(t_max, op=dist.ReduceOp.MAX)
    dist.all_reduce(t_sum, op=dist.ReduceOp.SUM)
    return float(t_max[0]), float(t_sum[0])


def make_cfg(w, layers=None, heads=None):
    from rolling_kv_cache_b200.cache import make_config
    return make_config(layers=w.layers if layers is None else layers,
                       heads=w.heads if heads is None else heads,
                       head_dim=w.head_dim, grid_h=w.grid_h, grid_w=w.grid_w,
                       sink_frames=w.sink_frames, window_frames=w.window_frames,
                       chunk_frames=w.chunk_frames, policy=w.policy,
                       mask_block_frames=w.mask_block_frames, theta=w.theta, t_max=w.t_max,
                       rs_bank_blocks=w.rs_bank_blocks, rs_sink_blocks=w.rs_sink_blocks,
                       rs_static_semantics=w.rs_static_semantics, ir_f_limit=w.ir_f_limit,
                       ir_sink_blocks=w.ir_sink_blocks, ir_cache_blocks=w.ir_cache_blocks,
                       df_budget_tokens=w.df_budget_tokens, rf_history_frames=w.rf_history_frames,
                       rf_weight=w.rf_weight, mr_alpha_long=w.mr_alpha_long,
                       mr_alpha_short=w.mr_alpha_short)


# ------------------------------------------------------------ CPU oracle
def oracle_sample_seconds(w, heads: int, chunk: int = 7):
    """Time the fp64 oracle on one layer-pass of a steady-state chunk,
    restricted to ``heads`` heads. Returns (seconds, flops, threads)."""
    from oracle import OracleStream
    st = OracleStream(w, layer=0, seed=0)
    rng = np.random.default_rng(0)   # Deep Forcing: the oracle's region follows given scores
    for c in range(chunk + 1):
        pool = rng.random(st.df.next_pool_size(w.chunk_frames)) if st.df is not None else None
        st.step(c, w.passes - 1 if c < chunk else 0, **({"pool_scores": pool} if st.df is not None else {}))
    st.outputs(heads=[0], rows=np.arange(1))       # warm the regenerated inputs
    t0 = time.perf_counter()
    st.outputs(heads=list(range(heads)))
    dt = time.perf_counter() - t0
    n_hist = sum(1 for k in st.kept_tokens if k.region != "cur") // w.frame_seqlen
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    return dt, attention_flops(w, n_hist, heads=heads), threads


def workload_config(w, world, shard, heads_per_rank):
    """The JSON line's ``config``: the same for both arms at the same N."""
    # bytes of one layer's K and V buffers (ring, plus the Deep Forcing region)
    kv_ring_mb = 2 * heads_per_rank * w.footprint_tokens * w.head_dim * 2 / 1e6
    return {"workload": w.name, "layers": w.layers, "heads": w.heads,
            "head_dim": w.head_dim, "frame_seqlen": w.frame_seqlen,
            "chunk_frames": w.chunk_frames, "sink_frames": w.sink_frames,
            "window_frames": w.window_frames, "passes_per_chunk": w.passes,
            "cached_tokens_per_head": w.footprint_tokens,
            "step": f"one chunk x {w.layers} layers x {w.passes} passes",
            "parallelism": (f"heads split over {world} GPUs (one stream)" if shard
                            else f"independent stream per GPU x{world}"),
            "l2": (f"inputs larger than L2 ({kv_ring_mb:.0f} MB K/V ring per layer"
                   f"{', %d layers cycled' % w.layers if w.layers > 1 else ''})")}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    heads = 1
    shard = args.shard == "heads"
    heads_per_rank = (w.heads + args.gpus - 1) // args.gpus if shard else w.heads
    for _ in range(args.warmup):
        oracle_sample_seconds(w, heads)
    secs, flops = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl, threads = oracle_sample_seconds(w, heads)
        secs += dt
        flops += fl
    value = flops / secs / 1e12
    sample = (f"fp64 numpy oracle, one head of one layer-pass per step (chunk 7 of {w.name}, "
              f"{w.query_tokens} queries x {steady_hist_frames(w) * w.frame_seqlen}+ keys)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.gpus, shard, heads_per_rank), "cpu_baseline": {
                "value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ GPU path
def nvtx_push(name):
    import torch
    try:
        torch.cuda.nvtx.range_push(name)
    except Exception:   # NVTX is a profiler annotation only
        pass


def nvtx_pop():
    import torch
    try:
        torch.cuda.nvtx.range_pop()
    except Exception:
        pass


def run_ours(args, w):
    import torch
    import torch.distributed as dist
    from rolling_kv_cache_b200 import binding as B
    from rolling_kv_cache_b200.cache import RollingKVCache
    from rolling_kv_cache_b200.shard import head_ranges, sharded_scores_topc

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    # --shard heads: this rank owns a head range of one stream (strong scaling);
    # default: an independent stream per rank (weak scaling)
    shard = args.shard == "heads"
    h0, h1 = head_ranges(w.heads, world)[rank] if shard else (0, w.heads)
    if h1 <= h0:
        raise SystemExit(f"--shard heads: rank {rank} of {world} would own no head of {w.heads}")
    cache = RollingKVCache(make_cfg(w, heads=h1 - h0), dev)
    stream = torch.cuda.current_stream(dev)
    # a small pool of distinct seeded inputs, resident in HBM, cycled over
    # (layer, pass, chunk); timing does not depend on the values
    pool = []
    for i in range(6):
        q, k, v = rc_synth.chunk_qkv(w, i % w.layers, i, i % w.passes, seed=0 if shard else rank)
        pool.append(tuple(torch.from_numpy(np.ascontiguousarray(x[:, h0:h1]).view(np.int16))
                          .view(torch.bfloat16).to(dev) for x in (q, k, v)))
    out = torch.empty_like(pool[0][0])
    B_ = w.chunk_frames
    calls_per_step = w.layers * w.passes
    # Deep-Forcing token scores + top-C on every step where the workload asks for them
    scores = torch.empty(w.footprint_tokens, dtype=torch.float32, device=dev) if w.topc else None
    topc = torch.empty(w.topc, dtype=torch.int32, device=dev) if w.topc else None

    def layer_step(l, q, k, v, frame_start, out_buf):
        if shard and scores is not None:
            # this rank's heads only; the score vectors are summed over ranks before top-C
            cache.step(l, q, k, v, frame_start, out=out_buf, scores=scores)
            sharded_scores_topc(cache, l, scores, w.topc, topc)
        else:
            cache.step(l, q, k, v, frame_start, out=out_buf, scores=scores, topc=topc, C=w.topc)

    def run_chunk(c, q_of=None, out_buf=None):
        if c in w.cut_chunks:   # KV flush + RoPE cut before the chunk's first pass
            cache.reindex(w.cut_delta, B.RC_REINDEX_FLUSH | B.RC_REINDEX_CUT)
        for p in range(w.passes):
            for l in range(w.layers):
                q, k, v = (q_of or pool)[(c * 7 + p * 3 + l) % len(q_of or pool)]
                layer_step(l, q, k, v, c * B_, out if out_buf is None else out_buf)

    chunk = 0
    # until the cache is full (the Deep / Relax Forcing region and MemRoPE memory included)
    prefill = (w.footprint_tokens // w.frame_seqlen + B_ - 1) // B_
    for _ in range(prefill):
        run_chunk(chunk)
        chunk += 1
    for _ in range(args.warmup):
        run_chunk(chunk)
        chunk += 1
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    B.rc_profile_begin(cache.handle, args.steps * calls_per_step * 6 + 16)
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    if not gpu_uuid.startswith("GPU-"):
        gpu_uuid = "GPU-" + gpu_uuid
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_uuid) as clocks:
        torch.cuda.synchronize()
        nvtx_push("timed")   # lets a profiler capture exactly the timed launches
        ev0.record(stream)
        for _ in range(args.steps):
            run_chunk(chunk)
            chunk += 1
        ev1.record(stream)
        torch.cuda.synchronize()
        nvtx_pop()
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    prof = B.rc_profile_end(cache.handle)
    cache.device_status()

    att = prof["attention"]
    ms_max, flops_total = aggregate_over_ranks(ms, att["flops"], dev)
    value = flops_total / (ms_max / 1e3) / 1e12
    frames = args.steps * B_ * world
    frames_per_s_per_layer = frames / (ms_max / 1e3) * w.layers / world
    launches = sum(v["launches"] for v in prof.values())

    # ---------------- end to end through the public API with host buffers
    e2e_steps = max(1, args.e2e_steps)
    host_pool = [tuple(t.cpu().pin_memory() for t in trip) for trip in pool[:3]]
    out_hosts = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * 2 for t in host_pool[0]) * calls_per_step
    d2h = out_hosts[0].numel() * 2 * calls_per_step
    pipe = cache.host_pipeline(depth=2)

    def e2e_step(chunk):
        fl = 0.0
        if chunk in w.cut_chunks:
            cache.reindex(w.cut_delta, B.RC_REINDEX_FLUSH | B.RC_REINDEX_CUT)
        for p in range(w.passes):
            for l in range(w.layers):
                q, k, v = host_pool[(p + l) % len(host_pool)]
                if shard and scores is not None:
                    pipe.submit(l, q, k, v, chunk * B_, out_hosts[pipe.i % 2], scores=scores)
                    sharded_scores_topc(cache, l, scores, w.topc, topc)
                else:
                    pipe.submit(l, q, k, v, chunk * B_, out_hosts[pipe.i % 2], scores=scores, topc=topc,
                                C=w.topc)
                st = cache.state(l)
                fl += 4.0 * w.head_dim * (h1 - h0) * visible_pairs(
                    w, sum(1 for e in st.kept[:st.n_kept] if e.region != 2) + st.comp_tokens // w.frame_seqlen)
        return fl

    # one untimed step first: the pipeline allocates its device staging
    # buffers on its first calls
    e2e_step(chunk)
    chunk += 1
    pipe.synchronize()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_flops = 0.0
    for _ in range(e2e_steps):
        e2e_flops += e2e_step(chunk)
        chunk += 1
    e1 = pipe.record_done()
    torch.cuda.synchronize()
    e2e_ms, e2e_tot = aggregate_over_ranks(e0.elapsed_time(e1), e2e_flops, dev)
    e2e_value = e2e_tot / (e2e_ms / 1e3) / 1e12

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    att_ms = att["ms"] / max(1, att["timed"])
    att_flops_launch = att["flops"] / max(1, att["launches"])
    achieved = att_flops_launch / (att_ms / 1e3) / 1e12
    # the committed capture covers one steady-state layer-pass of the Wan-1.3B stream
    traffic = attention_traffic() if w.name == "wan13b" else None
    app = prof["append"]
    app_gbs = (app["bytes"] / max(1, app["launches"])) / (app["ms"] / max(1, app["timed"]) / 1e3) / 1e9

    # the HBM-bound kernels at 40 heads (append, rotate-copy, in-place
    # re-rotation), each in its own single-layer stream after the timed region
    hbm = None
    if rank == 0 and not args.no_hbm:
        hbm = hbm_cases(dev, steps=10, warmup=2)
        hbm["append_12_heads"] = {"gbs": app_gbs, "frac": app_gbs / float(peaks.get("hbm_gbs", 6650.0)),
                                  "ms_per_launch": app["ms"] / max(1, app["timed"]),
                                  "bytes_per_launch": app["bytes"] / max(1, app["launches"]),
                                  "note": "inside the timed step above"}
    if world > 1:
        dist.barrier()

    # the attention's rate and the GEMM peak at the same SM clock: achieved
    # per MHz of the sampled median clock over the peak per MHz of the clock
    # the peak was measured at (when the peaks record it)
    clk = clocks.summary()
    peak_mhz = peak_clock_mhz(peaks, sustained=True)
    burst_mhz = peak_clock_mhz(peaks, sustained=False)
    sm_mhz = clk.get("sm_mhz")

    def per_clock(pk, mhz):
        if not mhz or not sm_mhz:
            return None
        return (achieved / sm_mhz) / (pk / mhz)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, fl, threads = oracle_sample_seconds(w, heads=3)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"fp64 numpy oracle, 3 of {w.heads} heads of one layer-pass at a "
                         f"steady-state chunk ({w.query_tokens} queries x "
                         f"{steady_hist_frames(w) * w.frame_seqlen}+ keys), {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "strong" if shard else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(w, world, shard, h1 - h0),
            "frames_per_s_per_layer": frames_per_s_per_layer,
            "frames_per_s_model": frames / (ms_max / 1e3),
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "path": "RollingKVCache.host_pipeline: pinned host q/k/v in, output back "
                            "to pinned host, uploads/downloads on their own streams overlapping "
                            "the kernels (depth 2)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "attention (tcgen05)",
                         "peak_source": f"{peak_src} bf16_tflops_sustained",
                         "frac_of_burst": achieved / float(peaks.get("bf16_tflops", peak)),
                         "frac_same_clock": per_clock(peak, peak_mhz),
                         "frac_of_burst_same_clock": per_clock(float(peaks.get("bf16_tflops", peak)), burst_mhz),
                         "clock_note": (f"attention at a median {sm_mhz} MHz; sustained peak at "
                                        f"{peak_mhz} MHz, burst peak at {burst_mhz} MHz "
                                        "(None: not recorded with the peaks)"),
                         "flops_per_launch": att_flops_launch, "ms_per_launch": att_ms},
            "kernels": {k: {"launches": v["launches"], "ms_per_launch": v["ms"] / max(1, v["timed"])}
                        for k, v in prof.items() if v["launches"]},
            "append_gbs": app_gbs, "append_hbm_frac": app_gbs / float(peaks.get("hbm_gbs", 6650.0)),
            "hbm": hbm,
            "gpu_launches": launches,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    cache.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


HBM_CASES = ("append", "rotcopy", "inplace")


def hbm_cases(dev, steps: int, warmup: int, only=HBM_CASES):
    """HBM-bound kernels at sizes where launch latency does not dominate.

    Three single-layer streams with 40 heads x 128 and 1560-token frames, run
    through rc_step; the library's per-launch CUDA events isolate the kernel:
      append    -- fused RoPE + append of a 3-frame chunk (287.5 MB per launch)
      rotcopy   -- Rolling Sink with static sink semantics: every step rotates
                   the 15 sink frames again from the raw bank (958 MB)
      inplace   -- sliding window with an 18-frame sink whose time index moves
                   by one every step: in-place time rotation (198 MB)
    Returns {case: {launches, ms_per_launch, bytes_per_launch, gbs, frac}}."""
    import torch
    from rolling_kv_cache_b200 import binding as B
    from rolling_kv_cache_b200.cache import RollingKVCache
    peaks, src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    base = rc_synth.WORKLOADS["large"]
    cases = {
        "append": (base, "append", None),
        "rotcopy": (rc_synth.WORKLOADS["rolling_sink"].replace(heads=40, rs_static_semantics=1,
                                                               dist="normal_frame_mean"), "rerotate", None),
        "inplace": (base.replace(sink_frames=18, window_frames=3), "rerotate", 1),
    }
    res = {}
    for name, (w, kind, sink_shift) in cases.items():
        if name not in only:
            continue
        cache = RollingKVCache(make_cfg(w, layers=1), dev)
        q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
                   for x in rc_synth.chunk_qkv(w, 0, 0, 0))
        out = torch.empty_like(q)
        chunk = 0

        def step():
            nonlocal chunk
            if sink_shift and chunk > 0:
                cache.reindex(sink_shift, B.RC_REINDEX_SINK)
            cache.step(0, q, k, v, chunk * w.chunk_frames, out=out)
            chunk += 1

        for _ in range(w.footprint_frames // w.chunk_frames + 1 + warmup):
            step()
        torch.cuda.synchronize()
        B.rc_profile_begin(cache.handle, 8 * steps + 16)
        for _ in range(steps):
            step()
        torch.cuda.synchronize()
        prof = B.rc_profile_end(cache.handle)[kind]
        ms = prof["ms"] / max(1, prof["timed"])
        by = prof["bytes"] / max(1, prof["launches"])
        gbs = by / (ms / 1e3) / 1e9
        res[name] = {"launches": prof["launches"], "ms_per_launch": ms, "bytes_per_launch": by,
                     "gbs": gbs, "frac": gbs / hbm}
        cache.close()
        del q, k, v, out
    res["peak_gbs"] = hbm
    res["peak_source"] = f"{src} hbm_gbs"
    res["config"] = {"heads": 40, "head_dim": 128, "frame_seqlen": 1560}
    return res


def run_hbm(args):
    """--hbm: only the HBM-bound kernels (see hbm_cases), one JSON line."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    only = [c for c in args.hbm_cases.split(",") if c] if args.hbm_cases else list(HBM_CASES)
    res = hbm_cases(dev, args.steps, args.warmup, only)
    print(json.dumps({"metric": "HBM GB/s of the append and re-rotation kernels", "unit": "GB/s",
                      "peak": res.pop("peak_gbs"), "peak_source": res.pop("peak_source"), "steps": args.steps,
                      "config": res.pop("config"), **res}), flush=True)
    return 0


def run_sdpa_context(args):
    """Context only (not the product path): torch's own scaled_dot_product_attention
    on the Wan-1.3B layer-pass shapes against this library's attention on the same
    shapes, both without an in-chunk mask (torch's fast kernels take no frame mask):
    one head-major [1, 12, 4680, 128] query block over [1, 12, 29640, 128] keys."""
    import torch
    import torch.nn.functional as Fn
    from rolling_kv_cache_b200 import binding as B
    from rolling_kv_cache_b200.cache import RollingKVCache
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = rc_synth.WORKLOADS["wan13b"].replace(layers=1, passes=1, mask_block_frames=3)
    H, d, Nq = w.heads, w.head_dim, w.query_tokens
    Nk = w.footprint_tokens
    flops = 4.0 * d * H * Nq * Nk

    def timed(fn, iters=20):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters

    g = torch.Generator(device=dev).manual_seed(0)
    q = torch.randn(1, H, Nq, d, device=dev, dtype=torch.bfloat16, generator=g)
    k = torch.randn(1, H, Nk, d, device=dev, dtype=torch.bfloat16, generator=g)
    v = torch.randn(1, H, Nk, d, device=dev, dtype=torch.bfloat16, generator=g)
    torch_res = {}
    from torch.nn.attention import SDPBackend, sdpa_kernel
    for name, be in (("cudnn", SDPBackend.CUDNN_ATTENTION), ("flash", SDPBackend.FLASH_ATTENTION),
                     ("efficient", SDPBackend.EFFICIENT_ATTENTION)):
        try:
            with sdpa_kernel([be]):
                ms = timed(lambda: Fn.scaled_dot_product_attention(q, k, v))
            torch_res[name] = {"ms": ms, "tflops": flops / (ms / 1e3) / 1e12}
        except Exception as e:   # backend not available for this shape / build
            torch_res[name] = {"unavailable": str(e).splitlines()[0][:120]}
    # this library, steady state of the same stream, the attention kernel's own events
    cache = RollingKVCache(make_cfg(w, layers=1), dev)
    pool = [tuple(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
                  for x in rc_synth.chunk_qkv(w, 0, c, 0)) for c in range(3)]
    out = torch.empty_like(pool[0][0])
    c = 0
    for _ in range((w.footprint_frames + 2) // 3 + 3):
        qq, kk, vv = pool[c % 3]
        cache.step(0, qq, kk, vv, 3 * c, out=out)
        c += 1
    torch.cuda.synchronize()
    B.rc_profile_begin(cache.handle, 256)
    for _ in range(20):
        qq, kk, vv = pool[c % 3]
        cache.step(0, qq, kk, vv, 3 * c, out=out)
        c += 1
    torch.cuda.synchronize()
    att = B.rc_profile_end(cache.handle)["attention"]
    ms = att["ms"] / max(1, att["timed"])
    ours = {"ms": ms, "tflops": att["flops"] / max(1, att["launches"]) / (ms / 1e3) / 1e12}
    cache.close()
    print(json.dumps({"metric": "context: attention TFLOP/s on the Wan-1.3B layer-pass shapes, no in-chunk mask",
                      "unit": "TFLOP/s", "queries": Nq, "keys": Nk, "heads": H, "head_dim": d,
                      "torch_sdpa": torch_res, "ours": ours}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan13b", choices=list(rc_synth.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--shard", choices=["streams", "heads"], default="streams",
                    help="streams: an independent stream per rank (weak scaling); heads: each rank "
                         "owns a head range of one stream, scores summed over ranks before top-C")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-hbm", action="store_true",
                    help="skip the HBM-bound kernel cases (40 heads) after the timed region")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (small profiling runs)")
    ap.add_argument("--sdpa-context", action="store_true",
                    help="context only: torch scaled_dot_product_attention vs this library on the same shapes")
    ap.add_argument("--hbm-cases", default="",
                    help="with --hbm: comma list of cases to run (append, rotcopy, inplace; default all)")
    ap.add_argument("--hbm", action="store_true",
                    help="measure the HBM-bound append / re-rotation kernels instead")
    args = ap.parse_args()
    if args.hbm:
        return run_hbm(args)
    if args.sdpa_context:
        return run_sdpa_context(args)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    w = rc_synth.WORKLOADS[args.workload]
    if args.layers:
        w = w.replace(layers=args.layers)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
