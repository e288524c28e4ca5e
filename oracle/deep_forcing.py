"""Deep Forcing token compaction: which tokens the cache keeps, at which time.

TEST INFRASTRUCTURE ONLY (see the package docstring). Plain Python integers.

rCM page, strategy 4 (Deep Forcing): instead of dropping whole blocks, the
cache is filtered token by token. Every layer scores each cached token by the
attention its key receives (q.k^T), and when the budget runs out it keeps
the deep sink (the first sink_frames frames), the top-C most important tokens
of the candidate range, and the recent tail (the last recent_frames frames).
After compaction, rope_time_delta_ rewrites the time encoding of the sink and
the compressed region in place, so that no empty time positions ("holes")
remain.

The page states the three kept parts and the in-place time fix and nothing
else; the readings taken (listed with reasons in the design notes):

DF1  Layout: deep sink (frames 0 .. S_f-1) + compressed region (at most C
     tokens) + recent tail (the newest W_f frames up to the end of the
     current chunk, the chunk included, as the sliding window reads W2).
DF2  When and from what: at a new chunk the tail drops its oldest frames E;
     the pool is the compressed region (in region order) followed by E's
     tokens (frame order, then token order). If the pool holds more than C
     tokens the region becomes the C highest-scoring pool tokens, ties to the
     lower pool index, kept in pool order (= time order). The scores are the
     Deep Forcing token scores of the last pass before the new chunk: the
     softmax mass each key received, summed over heads and queries (S1).
     Those tokens were all candidates of that pass (compressed region first,
     then the tail from its oldest frame), so the pool's scores are the first
     len(pool) candidate scores of that pass.
DF3  Budget: C is a whole number of frames' worth of tokens (C = V_max * F),
     so the region holds n_c = min(C, tokens dropped so far) tokens, a
     multiple of F.
DF4  Time indices without holes: tail and current frames keep tau = g (the
     absolute frame, as the sliding window). With g_t the first tail frame
     and V = n_c / F, region position i has tau = g_t - V + floor(i / F) and
     sink frame j has tau = g_t - V - S_f + j: sink, region and tail occupy
     consecutive time positions. Before anything has been dropped, V = 0 and
     g_t = S_f, so every frame sits at its own index. A token keeps its own
     (h, w) grid position.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

from .attention import top_c


@dataclasses.dataclass(frozen=True)
class KeptToken:
    """One key token of the cache, in logical order.

    content: stream frame whose raw k/v the token comes from.
    tok:     token index inside that frame (row-major h, w: reading W8).
    tau:     RoPE time index the key is rotated to.
    region:  "sink", "comp", "hist" (tail before the chunk) or "cur".
    rank:    chunk-relative frame of a "cur" token, -1 otherwise.
    """
    content: int
    tok: int
    tau: int
    region: str
    rank: int = -1


class DeepForcingOracle:
    """Full-history Deep Forcing cache for one layer (readings DF1-DF4)."""

    def __init__(self, chunk_frames: int, sink_frames: int, window_frames: int,
                 budget_tokens: int, frame_seqlen: int):
        if budget_tokens < 0 or budget_tokens % frame_seqlen:
            raise ValueError("the budget is a whole number of frames' worth of tokens (DF3)")
        if chunk_frames > window_frames:
            raise ValueError("chunk larger than the tail")
        self.B = chunk_frames
        self.S_f = sink_frames
        self.W_f = window_frames
        self.C = budget_tokens
        self.F = frame_seqlen
        self.end = 0
        self.cur_start: Optional[int] = None
        self.cur_n = 0
        self.comp: List[Tuple[int, int]] = []   # (frame, token) in region order
        self.last_pool: List[Tuple[int, int]] = []
        self.last_selection: Optional[np.ndarray] = None

    def tail_start(self, end: int) -> int:
        return max(self.S_f, end - self.W_f)

    def next_pool_size(self, n_frames: int) -> int:
        """Tokens in the pool of the next new chunk of n_frames frames."""
        dropped = self.tail_start(self.end + n_frames) - self.tail_start(self.end)
        return len(self.comp) + dropped * self.F

    def step(self, frame_start: int, n_frames: int,
             pool_scores: Optional[Sequence[float]] = None,
             selection: Optional[Sequence[int]] = None) -> List[KeptToken]:
        """Commit (or repeat) one chunk and return the kept key tokens.

        At a new chunk whose pool exceeds the budget, give either the pool's
        scores (DF2 selects from them) or the selection itself (ascending pool
        indices); a repeated ``frame_start`` (another pass) changes nothing.
        """
        if n_frames <= 0:
            raise ValueError("n_frames must be positive")
        if self.cur_start is not None and frame_start == self.cur_start:
            if n_frames != self.cur_n:
                raise ValueError("a repeated pass must cover the same frames")
        elif frame_start == self.end:
            old_t, new_t = self.tail_start(self.end), self.tail_start(frame_start + n_frames)
            dropped = [g for g in range(old_t, new_t) if g < self.end]
            pool = self.comp + [(g, t) for g in dropped for t in range(self.F)]
            self.last_pool = pool
            self.last_selection = None
            if len(pool) > self.C == 0:
                pool = []            # no budget: the region stays empty
            elif len(pool) > self.C:
                if selection is None:
                    if pool_scores is None or len(pool_scores) < len(pool):
                        raise ValueError("the pool exceeds the budget: give its scores or a selection")
                    selection = top_c(np.asarray(pool_scores[:len(pool)]), np.arange(len(pool)), self.C)
                selection = np.asarray(selection, dtype=np.int64)
                if (len(selection) != self.C or np.any(np.diff(selection) <= 0)
                        or selection[0] < 0 or selection[-1] >= len(pool)):
                    raise ValueError("a selection is C ascending pool indices")
                self.last_selection = selection
                pool = [pool[i] for i in selection]
            self.comp = pool
            self.end = frame_start + n_frames
            self.cur_start, self.cur_n = frame_start, n_frames
        else:
            raise ValueError("frame_start must repeat the last chunk or continue the stream")
        return self.kept()

    def kept(self) -> List[KeptToken]:
        """Key tokens in logical order with their time indices (DF4)."""
        F, g0, n = self.F, self.cur_start, self.cur_n
        end = g0 + n
        g_t = self.tail_start(end)
        V = len(self.comp) // F
        out = []
        for j in range(min(self.S_f, g0)):
            out += [KeptToken(j, t, g_t - V - self.S_f + j, "sink") for t in range(F)]
        for i, (g, t) in enumerate(self.comp):
            out.append(KeptToken(g, t, g_t - V + i // F, "comp"))
        for g in range(g_t, g0):
            out += [KeptToken(g, t, g, "hist") for t in range(F)]
        for g in range(g0, end):
            out += [KeptToken(g, t, g, "cur", g - g0) for t in range(F)]
        return out

    def frame_taus(self) -> Tuple[List[int], int, int]:
        """(sink frames' tau, first region tau, region virtual frames V)."""
        g0, n = self.cur_start, self.cur_n
        g_t = self.tail_start(g0 + n)
        V = len(self.comp) // self.F
        return [g_t - V - self.S_f + j for j in range(min(self.S_f, g0))], g_t - V, V
