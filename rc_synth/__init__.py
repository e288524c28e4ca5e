"""Seeded synthetic inputs for the chunked video-diffusion attention step.

This module is shared by the tests, the benchmark and the fp64 oracle. It holds
no arithmetic of the method (no RoPE, no eviction rule, no attention): only the
workload descriptions (sizes, policy knobs, stream schedule) and a
counter-based generator that turns a key
``(seed, workload, layer, chunk, pass, tensor)`` into the bf16 q/k/v tensors of
one call. Because every tensor can be regenerated from its key, a checker can
rebuild any frame of the stream's history without storing it.

Distributions follow the workloads the pages describe (Wan2.1-1.3B at 480x832,
LingBot-World 14B): standard normal values, optionally plus a mean shared by
all tokens of one latent frame (drawn per frame, head and channel with
standard deviation 0.5) to mimic frame redundancy. Values are drawn in fp32
and rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np

TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2

POLICY_NONE, POLICY_SLIDING, POLICY_ROLLING_SINK, POLICY_INFINITY_ROPE = 0, 1, 2, 3
POLICY_DEEP_FORCING = 4
POLICY_RELAX_FORCING = 5
POLICY_MEMROPE = 6


@dataclasses.dataclass(frozen=True)
class Workload:
    """One streamed workload: model-side sizes, cache policy and schedule."""

    name: str
    workload_id: int
    layers: int
    heads: int
    head_dim: int
    grid_h: int
    grid_w: int
    chunk_frames: int
    sink_frames: int
    window_frames: int
    policy: int
    chunks: int
    passes: int = 1
    dist: str = "normal"            # "normal" | "normal_frame_mean"
    # Rolling Sink: bank of K blocks, S of them feed the sink
    rs_bank_blocks: int = 0
    rs_sink_blocks: int = 0
    rs_static_semantics: int = 0
    # Infinity-RoPE
    ir_f_limit: int = 0
    ir_sink_blocks: int = 0
    ir_cache_blocks: int = 0
    cut_chunks: Tuple[int, ...] = ()
    cut_delta: int = 0
    # per-token scores + top-C on every step (0 = off)
    topc: int = 0
    # Deep Forcing: compressed-region budget in tokens (a multiple of the frame size)
    df_budget_tokens: int = 0
    # Relax Forcing: history frames kept between sink and tail, alignment weight
    rf_history_frames: int = 0
    rf_weight: float = 0.5
    # MemRoPE: EMA factors of the long- and short-term memory frames
    mr_alpha_long: float = 0.0
    mr_alpha_short: float = 0.0
    mask_block_frames: int = 1
    theta: float = 10000.0
    t_max: int = 4096

    @property
    def frame_seqlen(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def query_tokens(self) -> int:
        return self.chunk_frames * self.frame_seqlen

    @property
    def footprint_frames(self) -> int:
        return self.sink_frames + self.window_frames

    @property
    def footprint_tokens(self) -> int:
        mem = 2 if self.policy == POLICY_MEMROPE else 0
        return (self.footprint_frames + self.rf_history_frames + mem) * self.frame_seqlen + self.df_budget_tokens

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads. Frame grid 30x52 = 1560 tokens is the 480x832 latent
# (60x104 after the VAE, /4 after patching) the LingBot page works through.
WORKLOADS = {
    "tiny": Workload(
        name="tiny", workload_id=1, layers=1, heads=2, head_dim=64, grid_h=4,
        grid_w=4, chunk_frames=3, sink_frames=1, window_frames=6,
        policy=POLICY_SLIDING, chunks=10, passes=1, dist="normal"),
    "wan13b": Workload(
        name="wan13b", workload_id=2, layers=30, heads=12, head_dim=128,
        grid_h=30, grid_w=52, chunk_frames=3, sink_frames=1, window_frames=18,
        policy=POLICY_SLIDING, chunks=40, passes=5, dist="normal_frame_mean"),
    "large": Workload(
        name="large", workload_id=3, layers=1, heads=40, head_dim=128,
        grid_h=30, grid_w=52, chunk_frames=3, sink_frames=6, window_frames=12,
        policy=POLICY_SLIDING, chunks=120, passes=1, dist="normal_frame_mean"),
    "rolling_sink": Workload(
        name="rolling_sink", workload_id=4, layers=1, heads=12, head_dim=128,
        grid_h=30, grid_w=52, chunk_frames=3, sink_frames=15, window_frames=6,
        policy=POLICY_ROLLING_SINK, chunks=341, passes=1, dist="normal",
        rs_bank_blocks=6, rs_sink_blocks=5),
    "infinity_rope": Workload(
        name="infinity_rope", workload_id=5, layers=1, heads=12, head_dim=128,
        grid_h=30, grid_w=52, chunk_frames=3, sink_frames=3, window_frames=18,
        policy=POLICY_INFINITY_ROPE, chunks=100, passes=1, dist="normal",
        ir_f_limit=21, ir_sink_blocks=1, ir_cache_blocks=6,
        cut_chunks=(27, 60), cut_delta=21, topc=4680),
    # Deep Forcing (rCM page, strategy 4): deep sink 3 frames + a compressed
    # region of 12 frames' worth of tokens + recent tail of 6 frames (current
    # chunk included); same 32760-token footprint as the two block policies.
    "deep_forcing": Workload(
        name="deep_forcing", workload_id=6, layers=1, heads=12, head_dim=128,
        grid_h=30, grid_w=52, chunk_frames=3, sink_frames=3, window_frames=6,
        policy=POLICY_DEEP_FORCING, chunks=60, passes=1, dist="normal",
        df_budget_tokens=12 * 1560),
    # Relax Forcing (rCM page, strategy 5): sink 3 frames + 12 history frames
    # chosen by cosine similarity + tail of 6 frames; same 32760-token footprint.
    "relax_forcing": Workload(
        name="relax_forcing", workload_id=7, layers=1, heads=12, head_dim=128,
        grid_h=30, grid_w=52, chunk_frames=3, sink_frames=3, window_frames=6,
        policy=POLICY_RELAX_FORCING, chunks=60, passes=1, dist="normal_frame_mean",
        rf_history_frames=12, rf_weight=0.5),
    # MemRoPE (rCM page, MemRoPE tip): sink 3 + long/short EMA memory frames
    # + window 16 frames; same 32760-token footprint.
    "memrope": Workload(
        name="memrope", workload_id=8, layers=1, heads=12, head_dim=128,
        grid_h=30, grid_w=52, chunk_frames=3, sink_frames=3, window_frames=16,
        policy=POLICY_MEMROPE, chunks=60, passes=1, dist="normal_frame_mean",
        mr_alpha_long=0.9, mr_alpha_short=0.5),
}


def philox_key(seed: int, workload_id: int, layer: int, chunk: int,
               pass_: int, tensor_id: int) -> np.ndarray:
    """Pack the six key fields into Philox-4x64's two 64-bit key words."""
    for v, bits in ((workload_id, 16), (layer, 16), (pass_, 16), (tensor_id, 8)):
        if not 0 <= v < (1 << bits):
            raise ValueError("key field out of range")
    if not 0 <= chunk < (1 << 40) or not 0 <= seed < (1 << 32):
        raise ValueError("key field out of range")
    w0 = (seed << 32) | (workload_id << 16) | layer
    w1 = (chunk << 24) | (pass_ << 8) | tensor_id
    return np.array([w0, w1], dtype=np.uint64)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def chunk_tensor(w: Workload, layer: int, chunk: int, pass_: int, tensor_id: int,
                 seed: int = 0, n_frames: Optional[int] = None) -> np.ndarray:
    """bf16 bits of one of q/k/v for one call, shape [n_frames*F, H, d]."""
    nf = w.chunk_frames if n_frames is None else n_frames
    F = w.frame_seqlen
    g = np.random.Generator(np.random.Philox(
        key=philox_key(seed, w.workload_id, layer, chunk, pass_, tensor_id)))
    x = g.standard_normal((nf, F, w.heads, w.head_dim), dtype=np.float32)
    if w.dist == "normal_frame_mean":
        mean = g.standard_normal((nf, 1, w.heads, w.head_dim), dtype=np.float32)
        x += np.float32(0.5) * mean
    elif w.dist != "normal":
        raise ValueError(w.dist)
    return f32_to_bf16_bits(x.reshape(nf * F, w.heads, w.head_dim))


def chunk_qkv(w: Workload, layer: int, chunk: int, pass_: int, seed: int = 0):
    """(q, k, v) bf16 bits for one call."""
    return tuple(chunk_tensor(w, layer, chunk, pass_, t, seed)
                 for t in (TENSOR_Q, TENSOR_K, TENSOR_V))


def stream_schedule(w: Workload):
    """The call sequence of a workload: yields (chunk, pass, frame_start, cut).

    ``cut`` is True on the first pass of a chunk listed in ``cut_chunks``; the
    caller issues the flush + time cut before that call.
    """
    for c in range(w.chunks):
        for p in range(w.passes):
            yield c, p, c * w.chunk_frames, (p == 0 and c in w.cut_chunks)
