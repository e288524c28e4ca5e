"""Seeded input generator: determinism, bf16 rounding, distribution recipe."""
import numpy as np
import torch

import rc_synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-3, 3, 100000),
                        np.array([0.0, -0.0, 1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 65504.0], np.float32)])
    ours = rc_synth.f32_to_bf16_bits(x.astype(np.float32))
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = rc_synth.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_deterministic_and_keyed():
    w = rc_synth.WORKLOADS["tiny"]
    a = rc_synth.chunk_tensor(w, 0, 3, 0, rc_synth.TENSOR_K)
    b = rc_synth.chunk_tensor(w, 0, 3, 0, rc_synth.TENSOR_K)
    c = rc_synth.chunk_tensor(w, 0, 4, 0, rc_synth.TENSOR_K)
    d = rc_synth.chunk_tensor(w, 0, 3, 0, rc_synth.TENSOR_V)
    assert a.shape == (48, 2, 64) and a.dtype == np.uint16
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)


def test_frame_mean_recipe():
    w = rc_synth.WORKLOADS["wan13b"].replace(heads=4)
    x = rc_synth.bf16_bits_to_f32(rc_synth.chunk_tensor(w, 0, 0, 0, 0)).reshape(3, 1560, 4, 128)
    means = x.mean(axis=1)                     # per (frame, head, channel)
    assert abs(means.std() - 0.5) < 0.05       # shared per-frame mean, std 0.5
    resid = x - means[:, None]
    assert abs(resid.std() - 1.0) < 0.02       # N(0,1) per token
    y = rc_synth.bf16_bits_to_f32(rc_synth.chunk_tensor(rc_synth.WORKLOADS["rolling_sink"], 0, 0, 0, 0))
    assert abs(y.std() - 1.0) < 0.01 and abs(y.mean()) < 0.01


def test_schedule_and_sizes():
    w = rc_synth.WORKLOADS["wan13b"]
    sched = list(rc_synth.stream_schedule(w))
    assert len(sched) == 40 * 5 and sched[5] == (1, 0, 3, False)
    ir = rc_synth.WORKLOADS["infinity_rope"]
    cuts = [c for c, p, g, cut in rc_synth.stream_schedule(ir) if cut]
    assert cuts == [27, 60]
    assert w.query_tokens == 4680 and w.frame_seqlen == 1560
