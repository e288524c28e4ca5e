"""MemRoPE memory tokens: evicted frames folded into two EMA memory frames.

TEST INFRASTRUCTURE ONLY (see the package docstring). fp64 numpy.

rCM page, strategy 5's tip on MemRoPE: evicted frames are not dropped but
compressed into a long-term and a short-term memory by two exponential moving
averages (--mr_alpha_long / --mr_alpha_short); keys are stored raw and given
their position only when attention runs.

The page gives one sentence; the readings taken (listed with reasons in the
design notes):

MR1  Layout: sink (frames 0 .. S_f-1) + the two memory frames + window (the
     newest W_f frames up to the end of the current chunk, chunk included),
     as the sliding window with the memory in place of the evicted frames.
MR2  Update: every frame leaving the window, oldest first, is folded into
     both memories token by token (token i of a memory frame averages token
     i of the evicted frames), per head, for raw keys and values:
     M <- alpha * M + (1 - alpha) * X. The first evicted frame initialises
     both memories (M = X).
MR3  Position: at attention the long-term memory's keys are rotated to time
     S_f (right after the sink: the distant past) and the short-term
     memory's to g_w - 1 (right before the first window frame g_w: the
     recent past), each token at its own (h, w); every other frame keeps
     tau = g. Both are >= 0 whatever the sink size.
"""
from __future__ import annotations

from typing import Callable, List, Optional

import numpy as np

from .deep_forcing import KeptToken

MEM_LONG, MEM_SHORT = -1, -2   # "content" of the two memory frames


class MemRopeOracle:
    """Full-history MemRoPE cache for one layer (readings MR1-MR3).

    ``raw_frame(g, tid)`` returns frame g's raw k (tid 1) or v (tid 2),
    [F, H, d], of the last pass written.
    """

    def __init__(self, chunk_frames: int, sink_frames: int, window_frames: int,
                 alpha_long: float, alpha_short: float, frame_seqlen: int,
                 raw_frame: Callable[[int, int], np.ndarray]):
        if chunk_frames > window_frames:
            raise ValueError("chunk larger than the window")
        self.B, self.S_f, self.W_f, self.F = chunk_frames, sink_frames, window_frames, frame_seqlen
        self.alpha = {MEM_LONG: alpha_long, MEM_SHORT: alpha_short}
        self.raw_frame = raw_frame
        self.end = 0
        self.cur_start: Optional[int] = None
        self.cur_n = 0
        self.mem_k = {MEM_LONG: None, MEM_SHORT: None}
        self.mem_v = {MEM_LONG: None, MEM_SHORT: None}
        self.folded: List[int] = []   # evicted frames in folding order

    def window_start(self, end: int) -> int:
        return max(self.S_f, end - self.W_f)

    def step(self, frame_start: int, n_frames: int):
        if n_frames <= 0:
            raise ValueError("n_frames must be positive")
        if self.cur_start is not None and frame_start == self.cur_start:
            if n_frames != self.cur_n:
                raise ValueError("a repeated pass must cover the same frames")
        elif frame_start == self.end:
            new_end = frame_start + n_frames
            for g in range(self.window_start(self.end), self.window_start(new_end)):
                if g >= self.end:
                    break
                xk, xv = self.raw_frame(g, 1), self.raw_frame(g, 2)
                for m in (MEM_LONG, MEM_SHORT):
                    a = self.alpha[m]
                    if self.mem_k[m] is None:
                        self.mem_k[m], self.mem_v[m] = xk.copy(), xv.copy()
                    else:
                        self.mem_k[m] = a * self.mem_k[m] + (1.0 - a) * xk
                        self.mem_v[m] = a * self.mem_v[m] + (1.0 - a) * xv
                self.folded.append(g)
            self.end = new_end
            self.cur_start, self.cur_n = frame_start, n_frames
        else:
            raise ValueError("frame_start must repeat the last chunk or continue the stream")
        return self.kept()

    def kept(self) -> List[KeptToken]:
        F, g0, n = self.F, self.cur_start, self.cur_n
        end = g0 + n
        g_w = self.window_start(end)
        out = [KeptToken(g, t, g, "sink") for g in range(min(self.S_f, g0)) for t in range(F)]
        if self.folded:
            out += [KeptToken(MEM_LONG, t, self.S_f, "hist") for t in range(F)]
            out += [KeptToken(MEM_SHORT, t, g_w - 1, "hist") for t in range(F)]
        out += [KeptToken(g, t, g, "hist") for g in range(g_w, g0) for t in range(F)]
        out += [KeptToken(g, t, g, "cur", g - g0) for g in range(g0, end) for t in range(F)]
        return out

    def memory(self, which: int, tid: int) -> np.ndarray:
        """Raw k (tid 1) or v (tid 2) of a memory frame, [F, H, d]."""
        return (self.mem_k if tid == 1 else self.mem_v)[which]
