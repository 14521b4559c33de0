"""CPU oracle for a RoPE-compatible variant of store-h decode attention (test infrastructure
only, like ``storeh_oracle``; it shares no code with the CUDA library).

The pages describe store-h with K = W_k h exactly and say nothing about positional
encodings.  A model that uses rotary position embeddings rotates q and every K row by angles
that depend on their positions, which sits between the rebuild K = W_k h and the score, so the
absorbed form (one query vector per head applied to h) no longer holds for K: every cached row
needs its K rebuilt explicitly.  V is not rotated, so the value side keeps the absorbed form.

Readings (the pages are silent; the plainest standard form is taken):
1. Rotary embedding in the "rotate half" pairing of the head dimension: for a head vector x of
   head_dim hd at position t and i < hd/2, with theta_i = base^(-2i/hd),
       x'_i        = x_i cos(t theta_i) - x_{i+hd/2} sin(t theta_i)
       x'_{i+hd/2} = x_{i+hd/2} cos(t theta_i) + x_i sin(t theta_i)
   applied to q_j and to every K_cj, per head, after the projections; base = 10000 by default.
2. Positions: cached row c sits at position c (its cache index); the new token's query is at
   position ctx (its own row index), so a single query attends with relative offsets c - ctx.
3. Softmax scale 1/sqrt(hd), no biases, V = W_v h unrotated, as in the store-h decode.
"""
from __future__ import annotations

import math

import numpy as np


def rope_angles(positions: np.ndarray, hd: int, base: float) -> np.ndarray:
    """angles [n, hd/2] = position * base^(-2i/hd), in FP64."""
    i = np.arange(hd // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / hd)
    return np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]


def rotate(x: np.ndarray, positions: np.ndarray, hd: int, base: float) -> np.ndarray:
    """Rotary embedding (reading 1) of rows x [n, H * hd] at `positions` [n], per head, FP64."""
    n, d = x.shape
    H = d // hd
    a = rope_angles(positions, hd, base)
    c, s = np.cos(a)[:, None, :], np.sin(a)[:, None, :]
    xh = np.asarray(x, dtype=np.float64).reshape(n, H, hd)
    x1, x2 = xh[:, :, : hd // 2], xh[:, :, hd // 2:]
    out = np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=2)
    return out.reshape(n, d)


def attend_rope(h_hat: np.ndarray, h_new: np.ndarray, W_q: np.ndarray, W_k: np.ndarray, W_v: np.ndarray,
                H: int, hd: int, base: float = 10000.0, positions=None, q_position=None) -> np.ndarray:
    """Decode attention of one lane with rotary embeddings, K and V rebuilt explicitly.

    h_hat [n, d]: the dequantised rows 0..n-1 (row n-1 is the new token, appended first);
    positions default to 0..n-1 and the query's to n-1 (reading 2).  q = W_q h_new, K = W_k h,
    V = W_v h (FP64); q and K rotated; per head s_c = q'_j . K'_cj / sqrt(hd), p = softmax(s),
    o_j = sum_c p_c V_cj.  Returns o [H, hd]."""
    n, d = h_hat.shape
    assert d == H * hd
    pos = np.arange(n) if positions is None else np.asarray(positions)
    qpos = n - 1 if q_position is None else q_position
    Wq, Wk, Wv = (np.asarray(w, dtype=np.float64) for w in (W_q, W_k, W_v))
    q = Wq @ np.asarray(h_new, dtype=np.float64)
    K = h_hat @ Wk.T
    V = h_hat @ Wv.T
    qr = rotate(q[None, :], np.array([qpos]), hd, base)[0]
    Kr = rotate(K, pos, hd, base)
    out = np.empty((H, hd), dtype=np.float64)
    for j in range(H):
        cols = slice(j * hd, (j + 1) * hd)
        s = (Kr[:, cols] @ qr[cols]) / math.sqrt(hd)
        e = np.exp(s - np.max(s))
        out[j] = (e / np.sum(e)) @ V[:, cols]
    return out
