"""Which frames a bounded cache keeps, and at which RoPE time index.

TEST INFRASTRUCTURE ONLY (see the package docstring). Integer logic in plain
Python. Every step recomputes the kept set from the full history of the
stream; nothing is carried over from the previous step except the history
itself (frames committed so far, their virtual times, flush points).

Readings taken where the pages are silent or ambiguous are named by their
ids (W1..W7, D1, M1) and listed with their reasons in the design notes.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

POLICY_NONE, POLICY_SLIDING, POLICY_ROLLING_SINK, POLICY_INFINITY_ROPE = 0, 1, 2, 3
POLICY_DEEP_FORCING = 4   # token-level; see deep_forcing.py
POLICY_RELAX_FORCING = 5  # frame selection by similarity; see relax_forcing.py
POLICY_MEMROPE = 6        # EMA memory frames; see memrope.py

REINDEX_FLUSH = 1   # keep the sink and the last block, drop the middle
REINDEX_CUT = 2     # add t_delta to the virtual time of every later frame
REINDEX_SINK = 4    # add t_delta to the time index of the sink frames


@dataclasses.dataclass(frozen=True)
class KeptFrame:
    """One frame in the cache at a step, in logical order.

    content: stream frame index whose raw k/v the entry holds.
    tau:     RoPE time index (in latent frames) the entry is rotated to.
    region:  "sink", "hist" or "cur".
    rank:    chunk-relative frame index for "cur" entries, -1 otherwise.
    """
    content: int
    tau: int
    region: str
    rank: int = -1


def roll_index(p: int, K: int) -> int:
    """Bank block shown at block time p by Roll(x_[0,K)).

    Rolling Sink digest, method-step details: the K bank blocks are replayed
    cyclically, in forward order on even cycles and in reverse order on odd
    cycles. With period 2K and each end block repeated (0..K-1, K-1..0, ...),
    as reading W4 takes it.
    """
    if K <= 0 or p < 0:
        raise ValueError("roll_index needs K > 0 and p >= 0")
    q = p % (2 * K)
    return q if q < K else 2 * K - 1 - q


class PolicyOracle:
    """Full-history cache policy for one layer.

    Parameters mirror the library's cache config: ``chunk_frames`` is B (one
    block = one chunk), ``sink_frames``/``window_frames`` the footprint
    (reading W1: the sink sits inside the cache; the current chunk is part of
    the window, W2).
    """

    def __init__(self, policy: int, chunk_frames: int, sink_frames: int,
                 window_frames: int, rs_bank_blocks: int = 0,
                 rs_sink_blocks: int = 0, rs_static_semantics: int = 0,
                 ir_f_limit: int = 0, ir_sink_blocks: int = 0,
                 ir_cache_blocks: int = 0):
        self.policy = policy
        self.B = chunk_frames
        self.S_f = sink_frames
        self.W_f = window_frames
        self.K = rs_bank_blocks
        self.S = rs_sink_blocks
        self.rs_static = bool(rs_static_semantics)
        self.f_limit = ir_f_limit
        self.Sb = ir_sink_blocks
        self.Cb = ir_cache_blocks
        # history
        self.end = 0                  # frames committed so far
        self.cur_start: Optional[int] = None
        self.cur_n = 0
        self.vtime: List[int] = []    # virtual time of every committed frame
        self.cut_total = 0            # sum of cut deltas issued so far
        self.flush_points: List[int] = []   # stream frame where new content began
        self.sink_delta = 0           # sink-only time shift (REINDEX_SINK)
        self.last_kept: List[KeptFrame] = []

    @classmethod
    def from_workload(cls, w) -> "PolicyOracle":
        return cls(w.policy, w.chunk_frames, w.sink_frames, w.window_frames,
                   w.rs_bank_blocks, w.rs_sink_blocks, w.rs_static_semantics,
                   w.ir_f_limit, w.ir_sink_blocks, w.ir_cache_blocks)

    # ------------------------------------------------------------------ API
    def reindex(self, flags: int, t_delta: int) -> None:
        """Flush and/or time cut between chunks (rCM page, strategy 3, items 3-4).

        A flush keeps the global sink and the last committed block and drops
        the history in between (KV flush). A cut adds ``t_delta`` frames to
        the virtual time of everything committed afterwards (RoPE cut). Both
        take effect at the next new chunk (reading W7).
        """
        if flags & REINDEX_FLUSH:
            if self.policy != POLICY_INFINITY_ROPE:
                raise ValueError("flush is an Infinity-RoPE operation")
            self.flush_points.append(self.end)
        if flags & REINDEX_CUT:
            if self.policy != POLICY_INFINITY_ROPE:
                raise ValueError("cut is an Infinity-RoPE operation")
            self.cut_total += t_delta
        if flags & REINDEX_SINK:
            if self.policy not in (POLICY_SLIDING, POLICY_NONE):
                raise ValueError("sink shift applies to sliding / none")
            self.sink_delta += t_delta

    def step(self, frame_start: int, n_frames: int) -> List[KeptFrame]:
        """Commit (or overwrite) one chunk and return the kept frames.

        Repeated ``frame_start`` = another denoise pass of the same chunk: it
        overwrites the chunk in place and evicts nothing (LingBot page,
        sliding-window section: rolling fires only when the forward adds new
        content; reading D1).
        """
        if n_frames <= 0:
            raise ValueError("n_frames must be positive")
        if self.cur_start is not None and frame_start == self.cur_start:
            if n_frames != self.cur_n:
                raise ValueError("a repeated pass must cover the same frames")
        elif frame_start == self.end:
            self._check_new_chunk(frame_start, n_frames)
            for g in range(frame_start, frame_start + n_frames):
                self.vtime.append(g + self.cut_total)
            self.end = frame_start + n_frames
            self.cur_start, self.cur_n = frame_start, n_frames
        else:
            raise ValueError("frame_start must repeat the last chunk or continue the stream")
        kept = self._kept()
        self.last_kept = kept
        return kept

    # ------------------------------------------------------------ internals
    def _check_new_chunk(self, g0: int, n: int) -> None:
        if self.policy in (POLICY_ROLLING_SINK, POLICY_INFINITY_ROPE):
            if n != self.B or g0 % self.B:
                raise ValueError("block policies need whole blocks")
        if self.policy == POLICY_SLIDING and n > self.W_f:
            raise ValueError("chunk larger than the window")
        if self.policy == POLICY_NONE and g0 + n > self.S_f + self.W_f:
            raise ValueError("history exceeds the unbounded cache's capacity")

    def _kept(self) -> List[KeptFrame]:
        g0, n = self.cur_start, self.cur_n
        cur = range(g0, g0 + n)
        if self.policy == POLICY_NONE:
            return self._sliding(g0, n, window=self.end)
        if self.policy == POLICY_SLIDING:
            return self._sliding(g0, n, window=self.W_f)
        if self.policy == POLICY_ROLLING_SINK:
            return self._rolling_sink(g0)
        if self.policy == POLICY_INFINITY_ROPE:
            return self._infinity_rope(g0, n)
        raise ValueError("unknown policy")

    def _sliding(self, g0: int, n: int, window: int) -> List[KeptFrame]:
        """Sink + sliding window (LingBot page, local_attn_size and sink_size).

        The first S_f frames stay pinned; of the rest, the newest ``window``
        frames up to the end of the current chunk stay. RoPE takes the
        absolute frame number (LingBot page, two easily-missed details), so
        tau = g. Equivalently, num_evicted = new + used - capacity whole frames
        leave from just after the sink.
        """
        end = g0 + n
        out = []
        for g in range(min(self.S_f, end)):
            if g < g0:
                out.append(KeptFrame(g, g + self.sink_delta, "sink"))
        for g in range(max(self.S_f, end - window), g0):
            out.append(KeptFrame(g, g, "hist"))
        for g in range(g0, end):
            out.append(KeptFrame(g, g + (self.sink_delta if g < self.S_f else 0),
                                 "cur", g - g0))
        return out

    def _rolling_sink(self, g0: int) -> List[KeptFrame]:
        """Rolling Sink, stage 3 (Rolling Sink digest, method-step details).

        Step i generates block i conditioned on Cat(sink, x_[i-(K-S), i)).
        Sink time indices slide to [i-K, i-(K-S)); its content is a length-S
        segment of Roll(x_[0,K)), taken at the same positions (reading W4).
        With static semantics (stage 2) the sink shows blocks 0..S-1 at the
        sliding times.
        """
        B, K, S = self.B, self.K, self.S
        i = g0 // B
        out = []
        if i < K:
            for b in range(i):
                reg = "sink" if b < S else "hist"
                out += [KeptFrame(b * B + o, b * B + o, reg) for o in range(B)]
        else:
            for j, p in enumerate(range(i - K, i - K + S)):
                cb = j if self.rs_static else roll_index(p, K)
                out += [KeptFrame(cb * B + o, p * B + o, "sink") for o in range(B)]
            for b in range(i - (K - S), i):
                out += [KeptFrame(b * B + o, b * B + o, "hist") for o in range(B)]
        out += [KeptFrame(i * B + o, i * B + o, "cur", o) for o in range(B)]
        return out

    def _infinity_rope(self, g0: int, n: int) -> List[KeptFrame]:
        """Infinity-RoPE (rCM page, strategy 3).

        Kept: the global sink block(s), the last (cache_blocks - sink) blocks
        before the current one (reading W6), the current block; after a KV
        flush only the blocks from the one before the flush onwards. Time
        indices are block-relativistic: the newest block ends at f_limit
        (reading W5), everything shifts back by shift = max(0, G'_end -
        f_limit), and indices below 0 clamp to 0 (semanticization).
        """
        B = self.B
        sink_end = self.Sb * B
        lo = max(sink_end, g0 - (self.Cb - self.Sb) * B)
        flushes = [f for f in self.flush_points if f <= g0]
        if flushes:
            lo = max(lo, flushes[-1] - B)
        g_end_v = self.vtime[g0 + n - 1] + 1
        shift = max(0, g_end_v - self.f_limit)

        def tau(g):
            return max(0, self.vtime[g] - shift)

        out = [KeptFrame(g, tau(g), "sink") for g in range(min(sink_end, g0))]
        out += [KeptFrame(g, tau(g), "hist") for g in range(lo, g0)]
        out += [KeptFrame(g, tau(g), "cur", g - g0) for g in range(g0, g0 + n)]
        return out


def footprint_tokens(kept: List[KeptFrame], frame_seqlen: int) -> int:
    return len(kept) * frame_seqlen


def evicted_contents(prev: List[KeptFrame], new: List[KeptFrame]) -> List[int]:
    """Multiset difference of kept contents (previous step minus this one)."""
    from collections import Counter
    d = Counter(k.content for k in prev) - Counter(k.content for k in new)
    return sorted(d.elements())
