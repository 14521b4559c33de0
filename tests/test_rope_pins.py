"""Pins of the RoPE-variant oracle (no GPU) against things other than itself.

* the library's rotary embedding (transformers' Llama rotary module and apply_rotary_pos_emb)
  applied to explicitly stored K, attended by torch's scaled_dot_product_attention;
* relative positions only: shifting every position by the same amount changes nothing;
* a single row at position 0 is not rotated: the output is that row's V;
* without rotation (all positions 0) the variant is the store-h decode of the plain oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import rope_oracle


def _case(H=2, hd=16, n=9, seed=0):
    rng = np.random.default_rng(seed)
    d = H * hd
    W = [(rng.standard_normal((d, d)) / math.sqrt(d)).astype(np.float16) for _ in range(3)]
    h = rng.standard_normal((n, d)).astype(np.float16)
    return d, W, h


@pytest.mark.parametrize("H,hd,n,base", [(2, 16, 9, 10000.0), (4, 64, 31, 10000.0), (1, 128, 40, 500000.0)])
def test_matches_library_rotary_over_stored_kv(H, hd, n, base):
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
    d, W, h = _case(H, hd, n, seed=H + n)
    hh = h.astype(np.float64)
    got = rope_oracle.attend_rope(hh, h[-1], *W, H, hd, base=base)
    Wq, Wk, Wv = (torch.from_numpy(w.astype(np.float64)) for w in W)
    rows = torch.from_numpy(hh)
    K = torch.nn.functional.linear(rows, Wk).view(n, H, hd).permute(1, 0, 2).unsqueeze(0)
    V = torch.nn.functional.linear(rows, Wv).view(n, H, hd).permute(1, 0, 2).unsqueeze(0)
    q = torch.nn.functional.linear(torch.from_numpy(h[-1].astype(np.float64)), Wq).view(1, H, 1, hd)
    cfg = LlamaConfig(hidden_size=d, num_attention_heads=H, rope_theta=base, max_position_embeddings=4096)
    rot = LlamaRotaryEmbedding(config=cfg)
    cos, sin = rot(K, torch.arange(n)[None])
    # the query sits at the new token's position n - 1
    Kr, _ = apply_rotary_pos_emb(K, K, cos, sin)
    qr, _ = apply_rotary_pos_emb(q, q, cos[:, -1:], sin[:, -1:])
    want = torch.nn.functional.scaled_dot_product_attention(qr, Kr, V).view(H, hd).numpy()
    # the library evaluates its frequencies in fp32: angle errors up to n * 2^-24 rad
    assert np.max(np.abs(got - want)) < 1e-5, np.max(np.abs(got - want))


def test_shift_invariance():
    H, hd = 4, 64
    d, W, h = _case(H, hd, 23, seed=5)
    hh = h.astype(np.float64)
    a = rope_oracle.attend_rope(hh, h[-1], *W, H, hd)
    for shift in (1, 1000, 40000):
        b = rope_oracle.attend_rope(hh, h[-1], *W, H, hd, positions=np.arange(23) + shift, q_position=22 + shift)
        assert np.max(np.abs(a - b)) < 1e-9 * (1 + shift / 1000.0)


def test_single_row_at_position_zero_gives_its_v():
    H, hd = 2, 32
    d, W, h = _case(H, hd, 1, seed=8)
    o = rope_oracle.attend_rope(h.astype(np.float64), h[0], *W, H, hd)
    assert np.max(np.abs(o.reshape(-1) - W[2].astype(np.float64) @ h[0].astype(np.float64))) < 1e-13


def test_no_rotation_is_the_store_h_decode():
    H, hd = 4, 16
    d, W, h = _case(H, hd, 12, seed=9)
    hh = h.astype(np.float64)
    a = rope_oracle.attend_rope(hh, h[-1], *W, H, hd, positions=np.zeros(12), q_position=0)
    assert np.max(np.abs(a - oracle.attend_explicit(hh, h[-1], *W, H, hd))) < 1e-12


def test_rotation_matters():
    """The rotation changes the result (guards against a variant that never rotates)."""
    H, hd = 2, 16
    d, W, h = _case(H, hd, 12, seed=10)
    hh = h.astype(np.float64)
    a = rope_oracle.attend_rope(hh, h[-1], *W, H, hd)
    assert np.max(np.abs(a - oracle.attend_explicit(hh, h[-1], *W, H, hd))) > 1e-3
