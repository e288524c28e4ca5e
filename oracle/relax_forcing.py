"""Relax Forcing frame selection: which frames the cache keeps.

TEST INFRASTRUCTURE ONLY (see the package docstring). fp64 numpy for the
similarities, plain Python for the rest.

rCM page, strategy 5 (Relax Forcing): the cache is organised as Sink (global
anchor) + History (sparse history) + Tail (recent window). History frames
are chosen not by attention scores but by cosine similarity: each candidate
frame's alignment with the Tail region, plus a complementarity reward that
favours diversity, weighted as score = w * alignment + (1 - w) * complement,
and the Top-K frames kept. It selects whole frames, so it is cheaper than
Deep Forcing's per-token scores and the kept frames stay coherent in time.

The page gives the three parts and that formula; the readings taken (listed
with reasons in the design notes):

RF1  Layout: sink (frames 0 .. S_f-1) + history (at most K frames) + tail
     (the newest W_f frames up to the end of the current chunk, the chunk
     included). Every kept frame keeps tau = g, its absolute index, as the
     sliding window does (strategy 1): nothing is re-rotated.
RF2  Pool: at a new chunk the frames leaving the tail join the history
     frames; if the pool holds more than K frames, K are selected.
RF3  Descriptor of a frame: per head, the mean over the frame's tokens of
     its raw (unrotated) key, the heads concatenated (H * d values). The
     Tail descriptor is the mean of the descriptors of the tail's frames
     after the new chunk is appended (the chunk included).
RF4  alignment(f) = cos(desc(f), desc(Tail)).
RF5  complement(f) = 1 - the mean, over the other pool frames g, of
     cos(desc(f), desc(g)): a frame unlike the rest of the pool scores high.
RF6  score = w * alignment + (1 - w) * complement; the K highest scores are
     kept, ties to the older frame, in time order.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import numpy as np

from .policy import KeptFrame


def frame_descriptor(raw_k_frame: np.ndarray) -> np.ndarray:
    """RF3: mean over tokens of a frame's raw keys [F, H, d] -> [H * d]."""
    return np.asarray(raw_k_frame, dtype=np.float64).mean(axis=0).reshape(-1)


def cosine(a: np.ndarray, b: np.ndarray) -> float:
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0.0 or nb == 0.0:
        return 0.0
    return float(np.dot(a, b) / (na * nb))


def relax_scores(pool_desc: Sequence[np.ndarray], tail_desc: np.ndarray, weight: float) -> np.ndarray:
    """RF4-RF6 score of every pool frame."""
    n = len(pool_desc)
    align = np.array([cosine(d, tail_desc) for d in pool_desc])
    comp = np.ones(n)
    if n > 1:
        for i in range(n):
            comp[i] = 1.0 - sum(cosine(pool_desc[i], pool_desc[j]) for j in range(n) if j != i) / (n - 1)
    return weight * align + (1.0 - weight) * comp


def select_frames(scores: np.ndarray, K: int) -> List[int]:
    """RF6: indices of the K highest scores, ties to the lower index, ascending."""
    order = sorted(range(len(scores)), key=lambda i: (-scores[i], i))
    return sorted(order[:K])


class RelaxForcingOracle:
    """Full-history Relax Forcing cache for one layer (readings RF1-RF6).

    ``descriptor(g)`` returns frame g's RF3 descriptor (from its raw keys of
    the last pass written), supplied by the caller that holds the inputs.
    """

    def __init__(self, chunk_frames: int, sink_frames: int, window_frames: int,
                 history_frames: int, weight: float,
                 descriptor: Callable[[int], np.ndarray]):
        if chunk_frames > window_frames:
            raise ValueError("chunk larger than the tail")
        self.B = chunk_frames
        self.S_f = sink_frames
        self.W_f = window_frames
        self.K = history_frames
        self.w = weight
        self.descriptor = descriptor
        self.end = 0
        self.cur_start: Optional[int] = None
        self.cur_n = 0
        self.hist: List[int] = []            # selected history frames, ascending
        self.last_pool: List[int] = []
        self.last_scores: Optional[np.ndarray] = None
        self.last_selection: Optional[List[int]] = None

    def tail_start(self, end: int) -> int:
        return max(self.S_f, end - self.W_f)

    def step(self, frame_start: int, n_frames: int,
             selection: Optional[Sequence[int]] = None) -> List[KeptFrame]:
        """Commit (or repeat) one chunk; at a new chunk whose pool exceeds K
        the pool is scored (RF3-RF6) unless ``selection`` (ascending pool
        indices) is given."""
        if n_frames <= 0:
            raise ValueError("n_frames must be positive")
        if self.cur_start is not None and frame_start == self.cur_start:
            if n_frames != self.cur_n:
                raise ValueError("a repeated pass must cover the same frames")
        elif frame_start == self.end:
            new_end = frame_start + n_frames
            old_t, new_t = self.tail_start(self.end), self.tail_start(new_end)
            leaving = [g for g in range(old_t, new_t) if g < self.end]
            pool = self.hist + leaving
            self.last_pool = pool
            self.last_scores = None
            self.last_selection = None
            self.end = new_end
            self.cur_start, self.cur_n = frame_start, n_frames
            if len(pool) > self.K:
                if self.K == 0:
                    pool = []
                else:
                    descs = [self.descriptor(g) for g in pool]
                    tail = np.mean([self.descriptor(g) for g in range(new_t, new_end)], axis=0)
                    self.last_scores = relax_scores(descs, tail, self.w)
                    sel = list(selection) if selection is not None else select_frames(self.last_scores, self.K)
                    if len(sel) != self.K or sel != sorted(set(sel)) or sel[0] < 0 or sel[-1] >= len(pool):
                        raise ValueError("a selection is K ascending pool indices")
                    self.last_selection = sel
                    pool = [pool[i] for i in sel]
            self.hist = pool
        else:
            raise ValueError("frame_start must repeat the last chunk or continue the stream")
        return self.kept()

    def kept(self) -> List[KeptFrame]:
        g0, n = self.cur_start, self.cur_n
        end = g0 + n
        out = [KeptFrame(g, g, "sink") for g in range(min(self.S_f, g0))]
        out += [KeptFrame(g, g, "hist") for g in self.hist]
        out += [KeptFrame(g, g, "hist") for g in range(self.tail_start(end), g0)]
        out += [KeptFrame(g, g, "cur", g - g0) for g in range(g0, end)]
        return out
