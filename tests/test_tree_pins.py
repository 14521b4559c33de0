"""Pins of the tree-verification oracle (oracle/tree_oracle.py), no GPU.

* one branch of one token is the single-token decode of the store-h oracle;
* one branch of D tokens equals D sequential decodes, each over the cache grown by the
  branch's earlier tokens (the pages' "bit-identical to sequential generation");
* a token's output does not depend on the other branches (poisoned with NaN);
* permuting the branches permutes the outputs;
* the whole pass equals torch's library attention over the stacked rows with the tree mask.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import tree_oracle as T


def _case(seed, d=128, H=2, ctx=37, K=3, D=4, fmt=oracle.FMT_INT8):
    hd = d // H
    ctx_rows = synth.normal_f16(seed, 70, 0, ctx * d).reshape(ctx, d)
    tree_q = synth.normal_f16(seed, 71, 0, K * D * d).reshape(K, D, d)
    W = [synth.normal_f16(seed, 72 + i, 0, d * d, scale=1.0 / math.sqrt(d)).reshape(d, d) for i in range(3)]

    def stored(rows):
        codes, scales = oracle.quantize_rows(rows, fmt)
        return oracle.dequantize_rows(codes, scales, fmt, d)

    h_ctx = stored(ctx_rows)
    h_tree = stored(tree_q.reshape(K * D, d)).reshape(K, D, d)
    return h_ctx, h_tree, tree_q, W, H, hd


def test_single_token_is_the_decode():
    h_ctx, h_tree, q, W, H, hd = _case(1, K=1, D=1)
    out = T.tree_verify(h_ctx, h_tree, q, *W, H, hd)
    want = oracle.attend_explicit(np.concatenate([h_ctx, h_tree[0]]), q[0, 0], *W, H, hd)
    assert np.array_equal(out[0, 0], want)


def test_chain_equals_sequential_decodes():
    h_ctx, h_tree, q, W, H, hd = _case(2, K=1, D=5)
    out = T.tree_verify(h_ctx, h_tree, q, *W, H, hd)
    cache = h_ctx
    for t in range(5):
        cache = np.concatenate([cache, h_tree[0, t: t + 1]])  # the new token is appended, then attends
        assert np.array_equal(out[0, t], oracle.attend_explicit(cache, q[0, t], *W, H, hd)), t


def test_branches_do_not_see_each_other():
    h_ctx, h_tree, q, W, H, hd = _case(3)
    out = T.tree_verify(h_ctx, h_tree, q, *W, H, hd)
    for k in range(3):
        poisoned = h_tree.copy()
        poisoned[[j for j in range(3) if j != k]] = np.nan
        out_k = T.tree_verify(h_ctx, poisoned, q, *W, H, hd)[k]
        assert np.array_equal(out_k, out[k]), k


def test_branch_permutation():
    h_ctx, h_tree, q, W, H, hd = _case(4)
    perm = [2, 0, 1]
    out = T.tree_verify(h_ctx, h_tree, q, *W, H, hd)
    out_p = T.tree_verify(h_ctx, h_tree[perm], q[perm], *W, H, hd)
    assert np.array_equal(out_p, out[perm])


@pytest.mark.parametrize("K,D", [(1, 1), (1, 4), (4, 1), (3, 4)])
def test_matches_library_attention_with_the_tree_mask(K, D):
    h_ctx, h_tree, q, W, H, hd = _case(5 + K + D, K=K, D=D)
    d = h_ctx.shape[1]
    ctx = h_ctx.shape[0]
    Wq, Wk, Wv = (torch.from_numpy(w.astype(np.float64)) for w in W)
    rows = torch.from_numpy(np.concatenate([h_ctx, h_tree.reshape(K * D, d)]))
    Q = torch.nn.functional.linear(torch.from_numpy(q.reshape(K * D, d).astype(np.float64)), Wq)
    Kr = torch.nn.functional.linear(rows, Wk)
    Vr = torch.nn.functional.linear(rows, Wv)
    heads = lambda x: x.reshape(x.shape[0], H, hd).transpose(0, 1)  # [H, n, hd]
    mask = torch.from_numpy(T.tree_mask(ctx, K, D))
    lib = torch.nn.functional.scaled_dot_product_attention(heads(Q), heads(Kr), heads(Vr), attn_mask=mask)
    lib = lib.transpose(0, 1).reshape(K, D, H, hd).numpy()
    out = T.tree_verify(h_ctx, h_tree, q, *W, H, hd)
    assert np.max(np.abs(out - lib)) <= 1e-12 * max(1.0, np.max(np.abs(lib)))
