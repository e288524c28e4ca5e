"""The benchmark's FLOP count (the metric's numerator) against its definition.

Algorithmic FLOPs of a chunk's attention = 4 d H x (visible (query, key)
pairs); only the current chunk is masked. These checks count the pairs by
brute force from the oracle's visibility rule and pin the steady-state
layer-pass of the Wan-1.3B stream to its closed form.
"""
import numpy as np
import pytest

import bench
import rc_synth
from oracle import OracleStream
from oracle.attention import visibility

W = rc_synth.WORKLOADS


@pytest.mark.parametrize("name,mask_block", [("tiny", 1), ("tiny", 3), ("infinity_rope", 1),
                                             ("rolling_sink", 1), ("memrope", 1)])
def test_visible_pairs_match_brute_force(name, mask_block):
    w = W[name].replace(heads=1, grid_h=2, grid_w=3, mask_block_frames=mask_block)
    st = OracleStream(w)
    steady = w.footprint_tokens // w.frame_seqlen
    for c in range(steady):      # past the first eviction: the cache is full
        st.step(c, 0)
    F = w.frame_seqlen
    key_rank = np.array([k.rank for k in st.kept_tokens])
    q_rank = np.repeat(np.arange(w.chunk_frames), F)
    brute = int(visibility(q_rank, key_rank, mask_block).sum())
    n_hist = sum(1 for k in st.kept_tokens if k.region != "cur") // F
    assert bench.visible_pairs(w, n_hist) == brute


def test_wan13b_layer_pass_closed_form():
    w = W["wan13b"]
    F, H, d = w.frame_seqlen, w.heads, w.head_dim
    n_hist = bench.steady_hist_frames(w)
    assert n_hist == 16                       # sink 1 + window 18 - chunk 3
    # query frame r sees the 16 history frames and chunk frames 0..r
    pairs = sum(F * (n_hist * F + (r + 1) * F) for r in range(3))
    assert pairs == F * F * 54
    assert bench.attention_flops(w, n_hist) == 4.0 * d * H * pairs
    assert abs(bench.attention_flops(w, n_hist) / 1e12 - 0.8074) < 1e-4


def test_peak_clock_lookup():
    # the clock the GEMM peak was measured at, found wherever the peaks record it
    pk = {"hbm_gbs": 6557.8, "bf16_tflops": 1663.7, "bf16_tflops_sustained": 1390.4,
          "clocks": {"bf16_sustained": {"sm_mhz_median": 1342, "sm_mhz_max": 1965},
                     "bf16": {"sm_mhz_median": 1890}, "hbm_copy": {"sm_mhz_median": 1965, "mem_mhz": 3996}}}
    assert bench.peak_clock_mhz(pk, sustained=True) == 1342.0
    assert bench.peak_clock_mhz(pk, sustained=False) == 1890.0
    assert bench.peak_clock_mhz({"bf16_tflops": 1663.7}, sustained=True) is None


def test_traffic_needs_a_capture_of_the_current_source(tmp_path, monkeypatch):
    # the roofline's traffic is read from a capture summary only when that
    # capture was taken on the current attention kernel source
    import json
    import os
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.attention_traffic() is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    (prof / "attention_wan13b_ncu.json").write_text(json.dumps(
        {"kernel_source_sha256_16": "abc", "dram_bytes_per_launch": 2.5e8}))
    assert bench.attention_traffic() == 2.5e8
    (prof / "attention_wan13b_ncu.json").write_text(json.dumps(
        {"kernel_source_sha256_16": "old", "dram_bytes_per_launch": 2.5e8}))
    assert bench.attention_traffic() is None
    assert os.path.isdir(prof)
