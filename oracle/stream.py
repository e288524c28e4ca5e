"""Replays a workload's stream through the fp64 oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Keeps the whole history implicitly: raw q/k/v of any (chunk, pass) are
regenerated from their Philox key by ``rc_synth``, so the oracle can rotate
every kept frame from its raw values at its current time index (reading R3:
the oracle never composes rotations).
"""
from __future__ import annotations

from collections import OrderedDict
from typing import Dict, List, Optional, Sequence

import numpy as np

import rc_synth
from .policy import POLICY_DEEP_FORCING, POLICY_MEMROPE, POLICY_RELAX_FORCING, KeptFrame, PolicyOracle
from .deep_forcing import DeepForcingOracle, KeptToken
from .relax_forcing import RelaxForcingOracle, frame_descriptor
from .memrope import MemRopeOracle
from .rope import rope_angles, rope_apply, token_grid_positions
from .attention import column_scores, masked_sdpa, top_c, visibility


class OracleStream:
    """Integer state every step; fp64 outputs on request."""

    def __init__(self, w: "rc_synth.Workload", layer: int = 0, seed: int = 0,
                 cache_chunks: int = 16):
        self.w = w
        self.layer = layer
        self.seed = seed
        self.df = self.rf = self.mr = None
        if w.policy == POLICY_MEMROPE:
            self.policy = None
            self.mr = MemRopeOracle(w.chunk_frames, w.sink_frames, w.window_frames, w.mr_alpha_long,
                                    w.mr_alpha_short, w.frame_seqlen, self.frame_raw)
        elif w.policy == POLICY_DEEP_FORCING:
            self.policy = None
            self.df = DeepForcingOracle(w.chunk_frames, w.sink_frames, w.window_frames,
                                        w.df_budget_tokens, w.frame_seqlen)
        elif w.policy == POLICY_RELAX_FORCING:
            self.policy = self.rf = RelaxForcingOracle(
                w.chunk_frames, w.sink_frames, w.window_frames, w.rf_history_frames, w.rf_weight,
                lambda g: frame_descriptor(self.frame_raw(g, rc_synth.TENSOR_K)))
        else:
            self.policy = PolicyOracle.from_workload(w)
        self.last_pass: Dict[int, int] = {}
        self.cur = None
        self.kept: List[KeptFrame] = []
        self.kept_tokens: List[KeptToken] = []
        self._lru: "OrderedDict[tuple, np.ndarray]" = OrderedDict()
        self._lru_cap = 3 * cache_chunks

    # ------------------------------------------------------------ stream
    def reindex(self, flags: int, t_delta: int) -> None:
        if self.df is not None:
            raise ValueError("Deep Forcing has no reindex operation")
        self.policy.reindex(flags, t_delta)

    def step(self, chunk: int, pass_: int, pool_scores=None, selection=None):
        """Advance the policy; returns the kept frames (the kept key tokens
        under Deep Forcing, which takes the pool's scores or selection at a
        compaction: see DeepForcingOracle.step; Relax Forcing takes an
        optional selection, see RelaxForcingOracle.step)."""
        B = self.w.chunk_frames
        # this pass's raw values are what the cache holds from now on (D1)
        self.last_pass[chunk] = pass_
        if self.mr is not None:
            self.kept_tokens = self.mr.step(chunk * B, B)
            self.kept = []
        elif self.df is not None:
            self.kept_tokens = self.df.step(chunk * B, B, pool_scores, selection)
            self.kept = []
        elif self.rf is not None:
            self.kept = self.rf.step(chunk * B, B, selection)
            F = self.w.frame_seqlen
            self.kept_tokens = [KeptToken(k.content, t, k.tau, k.region, k.rank)
                                for k in self.kept for t in range(F)]
        else:
            self.kept = self.policy.step(chunk * B, B)
            F = self.w.frame_seqlen
            self.kept_tokens = [KeptToken(k.content, t, k.tau, k.region, k.rank)
                                for k in self.kept for t in range(F)]
        self.cur = (chunk, pass_)
        return self.kept_tokens if (self.df is not None or self.mr is not None) else self.kept

    # ------------------------------------------------------------ inputs
    def tensor(self, chunk: int, pass_: int, tid: int) -> np.ndarray:
        key = (chunk, pass_, tid)
        if key in self._lru:
            self._lru.move_to_end(key)
            return self._lru[key]
        bits = rc_synth.chunk_tensor(self.w, self.layer, chunk, pass_, tid, self.seed)
        val = rc_synth.bf16_bits_to_f32(bits).astype(np.float64)
        self._lru[key] = val
        if len(self._lru) > self._lru_cap:
            self._lru.popitem(last=False)
        return val

    def frame_raw(self, g: int, tid: int) -> np.ndarray:
        """Raw (unrotated) k or v of stream frame g, from its last pass."""
        B, F = self.w.chunk_frames, self.w.frame_seqlen
        c, o = divmod(g, B)
        t = self.tensor(c, self.last_pass[c], tid)
        return t[o * F:(o + 1) * F]

    # ----------------------------------------------------------- outputs
    def key_layout(self):
        """Per logical key token: tau, mask rank, region code (0 sink, 1
        history: compressed region and tail before the chunk, 2 current)."""
        kt = self.kept_tokens
        code = {"sink": 0, "comp": 1, "hist": 1, "cur": 2}
        tau = np.array([k.tau for k in kt], dtype=np.int64)
        rank = np.array([k.rank for k in kt], dtype=np.int64)
        region = np.array([code[k.region] for k in kt], dtype=np.int64)
        return tau, rank, region

    def _key_raw(self, tid: int) -> np.ndarray:
        """Raw k or v of every kept key token, in logical order."""
        kt = self.kept_tokens
        out, i = [], 0
        while i < len(kt):   # runs of tokens of one frame, gathered at once
            j = i
            while j + 1 < len(kt) and kt[j + 1].content == kt[i].content and kt[j + 1].region == kt[i].region:
                j += 1
            toks = np.array([k.tok for k in kt[i:j + 1]])
            src = self.mr.memory(kt[i].content, tid) if kt[i].content < 0 else self.frame_raw(kt[i].content, tid)
            out.append(src[toks])
            i = j + 1
        return np.concatenate(out)

    def outputs(self, heads: Optional[Sequence[int]] = None,
                rows: Optional[np.ndarray] = None, want_scores: bool = False):
        """fp64 attention of the current step.

        Returns dict with o [n_rows, n_heads, d], lse [n_heads, n_rows] and,
        with ``want_scores`` (all rows required), ``scores`` over candidate
        tokens, ``cand_index`` (their logical indices) and ``topc``.
        """
        w = self.w
        F, d = w.frame_seqlen, w.head_dim
        chunk, pass_ = self.cur
        heads = list(range(w.heads)) if heads is None else list(heads)
        nq = w.query_tokens
        rows = np.arange(nq) if rows is None else np.asarray(rows)
        if want_scores and len(rows) != nq:
            raise ValueError("scores need every query row")
        hh, ww = token_grid_positions(F, w.grid_w)
        cur_tau = {k.rank: k.tau for k in self.kept_tokens if k.region == "cur"}
        q_raw = self.tensor(chunk, pass_, rc_synth.TENSOR_Q)[rows]
        q_tau = np.array([cur_tau[r // F] for r in rows])
        q_rot = rope_apply(q_raw, rope_angles(q_tau, hh[rows % F], ww[rows % F], d, w.theta))

        k_tau, k_rank, region = self.key_layout()
        k_raw = self._key_raw(rc_synth.TENSOR_K)
        v_raw = self._key_raw(rc_synth.TENSOR_V)
        tok = np.array([k.tok for k in self.kept_tokens])
        k_rot = rope_apply(k_raw, rope_angles(k_tau, hh[tok], ww[tok], d, w.theta))
        vis = visibility(rows // F, k_rank, w.mask_block_frames)

        o = np.empty((len(rows), len(heads), d))
        lse = np.empty((len(heads), len(rows)))
        cand = np.nonzero(region == 1)[0]
        scores = None
        for i, h in enumerate(heads):
            oh, lh, p = masked_sdpa(q_rot[:, h], k_rot[:, h], v_raw[:, h], vis)
            o[:, i] = oh
            lse[i] = lh
            if want_scores:
                col = column_scores([p], cand)
                scores = col if scores is None else scores + col
            del p
        out = {"o": o, "lse": lse, "rows": rows, "heads": heads}
        if want_scores:
            if len(heads) != w.heads:
                raise ValueError("scores sum over every head")
            out["scores"] = scores
            out["cand_index"] = cand
            out["topc"] = top_c(scores, cand, w.topc)
        return out
