"""Masked scaled-dot-product attention, column scores and top-C in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).
"""
from __future__ import annotations

import numpy as np


def visibility(query_rank: np.ndarray, key_rank: np.ndarray,
               mask_block_frames: int = 1) -> np.ndarray:
    """Which keys each query sees: [n_q, n_k] bool.

    Only the current chunk is masked (reading M1): a cached key (rank -1) is
    visible to every query; a current-chunk key of chunk-relative frame r_k is
    visible to a query of frame r_q iff r_k // m <= r_q // m, with m =
    mask_block_frames (1 = frame-causal, = chunk size = no mask in the chunk).
    The frame-level block mask follows the Causal-Forcing page, section 2
    (num_frame_per_block: 1) and the rCM page's block mask tip.
    """
    qr = np.asarray(query_rank)[:, None] // mask_block_frames
    kr = np.asarray(key_rank)[None, :]
    return (kr < 0) | ((kr // mask_block_frames) <= qr)


def masked_sdpa(q: np.ndarray, k: np.ndarray, v: np.ndarray, visible: np.ndarray):
    """softmax(q k^T / sqrt(d) + mask) v for one head, fp64.

    q [n_q, d], k [n_k, d], v [n_k, d], visible [n_q, n_k]. Returns
    (o [n_q, d], lse [n_q] natural-log logsumexp of the scaled scores,
    p [n_q, n_k] probabilities). Scale 1/sqrt(d) (reading S2).
    """
    d = q.shape[1]
    s = (q @ k.T) / np.sqrt(np.float64(d))
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    return p @ v, (np.log(l) + m)[:, 0], p


def column_scores(p_per_head, candidate_cols: np.ndarray) -> np.ndarray:
    """Deep Forcing token score: attention mass each cached token receives.

    rCM page, strategy 4: each layer scores every cached token by its q.k^T
    attention. Reading S1: the score of key j is the sum over heads and over
    the current chunk's queries of the softmax probability p[h, q, j] that
    the attention actually used.
    """
    total = None
    for p in p_per_head:
        col = p[:, candidate_cols].sum(axis=0)
        total = col if total is None else total + col
    return total


def top_c(scores: np.ndarray, logical_index: np.ndarray, C: int) -> np.ndarray:
    """The C highest-scoring tokens, ties to the lower logical index.

    Returned as ascending logical indices (rCM page, strategy 4: keep the
    top-C important tokens of the candidate range).
    """
    scores = np.asarray(scores)
    logical_index = np.asarray(logical_index)
    order = np.lexsort((logical_index, -scores))
    return np.sort(logical_index[order[:min(C, len(order))]])
