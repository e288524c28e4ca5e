"""3D (t, h, w) rotary position embedding in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages fix that queries and keys carry a 3D RoPE over time, row and column
(Causal-Forcing page, section 3: causal_rope_apply with start_frame gives new
frames their absolute time; LingBot page, two easily-missed details: RoPE
takes the absolute frame number; Rolling Sink digest, RoPE background: each
frequency dimension rotates at its own speed). They are silent on pairing,
frequencies and axis order; readings R1/R2 take:

* c = d/2 rotation pairs split P_t = c - 2*floor(c/3), P_h = P_w = floor(c/3)
  (d=128: 22/21/21 pairs = 44/42/42 dims; d=64: 12/10/10 pairs);
* pairs are adjacent elements (2m, 2m+1), ordered t, then h, then w;
* axis frequencies omega_j = theta^(-2j / (2 P_axis)), j = 0..P_axis-1;
* (x, y) -> (x cos a - y sin a, x sin a + y cos a) with a = pos * omega_j.
"""
from __future__ import annotations

import numpy as np


def rope_pair_split(head_dim: int):
    """(P_t, P_h, P_w) rotation pairs per axis for a head dimension."""
    if head_dim % 2:
        raise ValueError("head_dim must be even")
    c = head_dim // 2
    p_hw = c // 3
    return c - 2 * p_hw, p_hw, p_hw


def axis_frequencies(n_pairs: int, theta: float) -> np.ndarray:
    j = np.arange(n_pairs, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * j / (2.0 * n_pairs))


def token_grid_positions(frame_seqlen: int, grid_w: int):
    """(row, col) of each token of a frame, row-major (reading W8)."""
    n = np.arange(frame_seqlen)
    return n // grid_w, n % grid_w


def rope_angles(t_pos, h_pos, w_pos, head_dim: int, theta: float) -> np.ndarray:
    """Rotation angle of every pair for every token: [n_tokens, d/2] fp64."""
    pt, ph, pw = rope_pair_split(head_dim)
    t_pos = np.asarray(t_pos, dtype=np.float64)
    h_pos = np.asarray(h_pos, dtype=np.float64)
    w_pos = np.asarray(w_pos, dtype=np.float64)
    return np.concatenate([
        np.outer(t_pos, axis_frequencies(pt, theta)),
        np.outer(h_pos, axis_frequencies(ph, theta)),
        np.outer(w_pos, axis_frequencies(pw, theta)),
    ], axis=1)


def rope_apply(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate x [n_tokens, H, d] (fp64) by per-token pair angles [n_tokens, d/2]."""
    x = np.asarray(x, dtype=np.float64)
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out
