"""CPU oracle for multi-query (tree) verification over the store-h cache (test
infrastructure only, like ``storeh_oracle``; it shares no code with the CUDA library).

What it computes [Architecture-Exclusive Features, "Tree speculative decoding"]: K draft
branches, each a chain of D tokens grown from the same root (the lane's last accepted
token), are verified in one mask-gated attention pass over the lane's cache.  Token (k, t)
of the tree attends the lane's cached positions 0..ctx-1 and the tree tokens (k, 0..t) of its
own branch, itself included, and nothing of the other branches.  With one branch (K = 1) the
pass equals D sequential single-token decodes, which is the pages' "bit-identical to
sequential generation" claim.

Readings (the pages give the tree shape and the mask only in words):
1. The tree tokens' own rows are appended to the cache first and read back in the cache's
   format, like the single new token of a decode; the queries come from their unquantised
   fp16 states.
2. The tree is K independent chains from the root (top-K at the root, then chain extension),
   so the mask is causal within a branch and empty across branches.
"""
from __future__ import annotations

import numpy as np

from .storeh_oracle import attend_explicit


def tree_rows(h_ctx: np.ndarray, h_tree: np.ndarray, k: int, t: int) -> np.ndarray:
    """The rows token (k, t) attends: the cached rows, then tokens 0..t of branch k."""
    return np.concatenate([h_ctx, h_tree[k, : t + 1]], axis=0)


def tree_verify(h_ctx: np.ndarray, h_tree: np.ndarray, h_query: np.ndarray, W_q: np.ndarray, W_k: np.ndarray,
                W_v: np.ndarray, H: int, hd: int) -> np.ndarray:
    """Outputs of every tree token.

    h_ctx [ctx, d]: the lane's cached rows (dequantised); h_tree [K, D, d]: the tree tokens'
    rows as the cache holds them (dequantised); h_query [K, D, d]: their unquantised fp16
    states, which form the queries.  Returns out [K, D, H, hd] in FP64."""
    K, D, d = h_tree.shape
    out = np.empty((K, D, H, hd), dtype=np.float64)
    for k in range(K):
        for t in range(D):
            out[k, t] = attend_explicit(tree_rows(h_ctx, h_tree, k, t), h_query[k, t], W_q, W_k, W_v, H, hd)
    return out


def tree_mask(ctx: int, K: int, D: int) -> np.ndarray:
    """Boolean [K*D, ctx + K*D] mask of the pass over the stacked rows (cache, then the tree
    tokens branch by branch): True where query (k, t) may attend."""
    M = K * D
    m = np.zeros((M, ctx + M), dtype=bool)
    m[:, :ctx] = True
    for k in range(K):
        for t in range(D):
            m[k * D + t, ctx + k * D: ctx + k * D + t + 1] = True
    return m
